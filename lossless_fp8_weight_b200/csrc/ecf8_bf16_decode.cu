// GPU decoder of the BF16 variant (DFloat11 article §2-§3: the exponent
// field Huffman-coded per tensor over 256 values, sign and mantissa kept as
// one byte; blob layout as in bf16_oracle.c / ecf8_bf16_host.cpp).
//
// The same plan as the ECF8 decoder, with an 8-bit alphabet: one warp per
// group of 32 chunks of 32 stream bytes; each lane shifts its slice to its
// first code (the gap), zeroes the bits after its last code and walks 68
// nibbles through a state machine (256 tree nodes x 16 nibbles, 64-bit
// entries: the exponents that end in the nibble and the next node; the table
// comes from the host, ecf8_bf16_build_table); zero-padding codes are
// subtracted; a warp scan places each lane's exponents; they are packed a
// byte each into lane-private shared memory, funnel-shifted into a byte stage,
// and 16 exponents plus 16 kept bytes become 16 BF16 values per lane step.
// Corrupt input is reported through the status word; no access leaves its
// buffer and no loop runs without a bound.
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "ecf8.h"
#include "ecf8_format.h"

namespace ecf8_bf16 {
namespace {

constexpr int kC = 32, kT = 32;
constexpr int kWords = kC / 4;               // stream words per chunk
constexpr int kSpanBits = 8 * kC;            // 256
constexpr int kNibbles = 68;                 // 272 bits: a lane may own up to 256 + 15 bits
constexpr int kPadBits = 4 * kNibbles;
constexpr int kPrivWords = kNibbles + 1;     // <= 272 codes, 4 per word
constexpr int kMaxCodes = kSpanBits * kT;    // 8192
constexpr int kStageWords = kMaxCodes / 4 + 8;
constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr uint32_t kErr = 255;

struct alignas(16) WarpArea {
  uint32_t priv[kPrivWords * 32];  // word k of lane l at k*32 + l
  uint32_t stage[kStageWords];     // exponent byte i at byte i (from the group's 16-aligned base)
};
struct alignas(16) Smem {
  uint2 table[256 * 16];  // (node << 4 | nibble) -> {exponents, next node << 4 | 8*count << 12}
  uint16_t zero_codes[kPadBits + 1];
  uint16_t pad_[7];
  WarpArea warp[kWarps];
};
static_assert(offsetof(Smem, warp) % 16 == 0, "warp areas must be 16-byte aligned");
static_assert(offsetof(WarpArea, stage) % 16 == 0, "stage must be 16-byte aligned");
static_assert(sizeof(Smem) <= 227 * 1024, "shared memory budget");

struct Args {
  const uint32_t* gaps;
  const uint64_t* groups;
  const uint32_t* stream;
  const uint8_t* kept;
  uint16_t* out;
  uint64_t n, code_bits;
  uint32_t n_groups, lmin;
};

struct GroupIn {
  uint32_t w[kWords + 1];
  uint32_t gapw, gapn;
  uint64_t off0, off1;
};

__device__ __forceinline__ void fetch_group(const Args& a, uint32_t g, GroupIn& in) {
  const uint32_t lane = threadIdx.x & 31;
  const uint64_t chunk = (uint64_t)g * kT + lane;
  const uint4* cs = reinterpret_cast<const uint4*>(a.stream + chunk * kWords);
#pragma unroll
  for (int q = 0; q < kWords / 4; ++q) {
    const uint4 v = __ldg(cs + q);
    in.w[4 * q + 0] = v.x;
    in.w[4 * q + 1] = v.y;
    in.w[4 * q + 2] = v.z;
    in.w[4 * q + 3] = v.w;
  }
  in.w[kWords] = __ldg(a.stream + (chunk + 1) * kWords);
  in.gapw = __ldg(a.gaps + (chunk >> 3));
  in.gapn = (lane == 31 && g + 1 < a.n_groups) ? __ldg(a.gaps + ((chunk + 1) >> 3)) : 0u;
  in.off0 = __ldg(a.groups + g);
  in.off1 = __ldg(a.groups + g + 1);
}

// BF16 pair from two exponents (bits 0-7, 16-23 of q) and two kept bytes
// (bits 0-7, 16-23 of p): kept + exponent * 128 + sign * 255 * 128 puts the
// sign at bit 15 and the exponent at bits 7-14 without carries between halves.
__device__ __forceinline__ uint32_t pair_bf16(uint32_t p, uint32_t q) {
  return p + q * 128u + (p & 0x00800080u) * 255u;
}

__device__ void process_group(const Args& a, uint32_t g, const GroupIn& in, const Smem* sm, WarpArea* wa,
                              int32_t* status) {
  const uint32_t lane = threadIdx.x & 31;
  const uint64_t off0 = in.off0, off1 = in.off1;
  const bool offsets_ok = off0 <= off1 && off1 <= a.n && off1 - off0 <= (uint64_t)kMaxCodes;

  // the lane's bits run from its first code to the next lane's first code or the stream end
  const uint32_t gap = (in.gapw >> ((lane & 7) * 4)) & 15u;
  uint32_t gap_next = __shfl_down_sync(0xFFFFFFFFu, gap, 1);
  if (lane == 31) gap_next = in.gapn & 15u;
  const uint64_t bit0 = ((uint64_t)g * kT + lane) * kSpanBits;
  const uint64_t left = bit0 < a.code_bits ? a.code_bits - bit0 : 0;
  const uint32_t stop = left < (uint64_t)(kSpanBits + gap_next) ? (uint32_t)left : kSpanBits + gap_next;
  const uint32_t E = stop > gap ? stop - gap : 0;
  uint32_t sw[kWords + 1];
#pragma unroll
  for (int i = 0; i < kWords; ++i) sw[i] = __funnelshift_l(in.w[i + 1], in.w[i], gap);
  sw[kWords] = in.w[kWords] << gap;
#pragma unroll
  for (int i = 0; i <= kWords; ++i) {
    const int keep = min(max((int)E - 32 * i, 0), 32);
    sw[i] &= (uint32_t)(0xFFFFFFFF00000000ull >> keep);
  }

  // the nibble machine: 68 steps, exponents packed a byte each
  uint32_t* priv = wa->priv + lane;
  uint32_t y = 0, acc = 0, sh = 0, words = 0;
#pragma unroll
  for (int j = 0; j < kNibbles; ++j) {
    const uint32_t nib = (sw[j >> 3] >> (28 - 4 * (j & 7))) & 15u;
    const uint2 e = sm->table[(y & 0xFF0u) | nib];
    y = e.y;
    acc |= e.x << sh;
    const uint32_t carry = __funnelshift_l(e.x, 0u, sh);
    sh += e.y >> 12;
    if (sh >= 32) {
      if (words < (uint32_t)kPrivWords) priv[32 * words] = acc;
      ++words;
      acc = carry;
      sh -= 32;
    }
  }
  if (sh && words < (uint32_t)kPrivWords) priv[32 * words] = acc;
  const uint32_t emitted = 4 * words + sh / 8;
  const uint32_t extra = sm->zero_codes[kPadBits - (E < (uint32_t)kPadBits ? E : (uint32_t)kPadBits)];
  const bool bad = ((y >> 4) & 0xFFu) == kErr || emitted < extra || words > (uint32_t)kPrivWords;
  const uint32_t cnt = bad ? 0 : emitted - extra;

  uint32_t incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= (uint32_t)o) incl += v;
  }
  const uint32_t total = __shfl_sync(0xFFFFFFFFu, incl, 31);
  const uint32_t start = incl - cnt;
  const bool any_bad = __any_sync(0xFFFFFFFFu, bad);
  if (any_bad || !offsets_ok || (uint64_t)total != off1 - off0) {
    if (lane == 0 && status) {
      int32_t f = 0;
      if (any_bad) f |= ECF8_STATUS_BAD_CODE;
      if (!offsets_ok) f |= ECF8_STATUS_BAD_OFFSETS;
      else if ((uint64_t)total != off1 - off0) f |= ECF8_STATUS_COUNT_MISMATCH;
      atomicOr(status, f);
    }
    return;
  }

  // exponent bytes into the stage at byte (off0 mod 16) + start
  uint32_t* stage = wa->stage;
  const uint32_t q = (uint32_t)(off0 & 15) + start;
  const uint32_t d0 = q >> 2, dl = cnt ? (q + cnt - 1) >> 2 : 0;
  if (cnt) {
    stage[d0] = 0;
    stage[dl] = 0;
  }
  __syncwarp();
  if (cnt) {
    const uint32_t r = (q & 3) * 8;
    const uint32_t used = (cnt + 3) / 4;
    if (cnt & 3) priv[32 * (used - 1)] &= (1u << (8 * (cnt & 3))) - 1;
    const uint32_t nwd = dl - d0 + 1;
    uint32_t prev = priv[0];
    atomicOr(&stage[d0], prev << r);
    uint32_t j = 1;
    for (; j + 1 < nwd; ++j) {
      const uint32_t cur = priv[32 * j];
      stage[d0 + j] = __funnelshift_l(prev, cur, r);
      prev = cur;
    }
    if (nwd > 1) {
      const uint32_t cur = j < used ? priv[32 * j] : 0;
      atomicOr(&stage[d0 + j], __funnelshift_l(prev, cur, r));
    }
  }
  __syncwarp();

  // 16 weights per lane step: 16 exponent bytes + 16 kept bytes -> 32 output bytes
  const uint64_t base = off0 & ~15ull;
  const uint32_t units = (uint32_t)(((off0 & 15) + (off1 - off0) + 15) >> 4);
  const uint32_t first_full = (off0 & 15) ? 1u : 0u;
  const uint32_t end_full = (units && (off1 & 15)) ? units - 1 : units;
  const uint4* st = reinterpret_cast<const uint4*>(stage);
  for (uint32_t u = lane; u < end_full; u += 32) {
    if (u < first_full) continue;
    const uint4 ex = st[u];
    const uint4 kb = __ldg(reinterpret_cast<const uint4*>(a.kept + base) + u);
    const uint32_t e4[4] = {ex.x, ex.y, ex.z, ex.w}, k4[4] = {kb.x, kb.y, kb.z, kb.w};
    uint32_t o[8];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      o[2 * w] = pair_bf16(__byte_perm(k4[w], 0u, 0x4140), __byte_perm(e4[w], 0u, 0x4140));
      o[2 * w + 1] = pair_bf16(__byte_perm(k4[w], 0u, 0x4342), __byte_perm(e4[w], 0u, 0x4342));
    }
    uint4* dst = reinterpret_cast<uint4*>(a.out + base + 16ull * u);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
  // the ragged first and last unit, one weight per lane (lanes 0-15 head, 16-31 tail)
  const bool hr = units && first_full;
  const bool tr = end_full < units && !(hr && end_full == 0);
  const bool rg = lane < 16 ? hr : tr;
  const uint32_t ru = lane < 16 ? 0u : end_full;
  const uint64_t p = base + 16ull * ru + (lane & 15);
  if (rg && p >= off0 && p < off1) {
    const uint32_t i = 16 * ru + (lane & 15);
    const uint32_t e = (stage[i >> 2] >> (8 * (i & 3))) & 0xFFu;
    const uint32_t k = a.kept[p];
    a.out[p] = (uint16_t)(((k >> 7) << 15) | (e << 7) | (k & 0x7Fu));
  }
  __syncwarp();
}

__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const uint2* __restrict__ d_table, Args a,
                                                              int32_t* status) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Smem* sm = reinterpret_cast<Smem*>(smem_raw);
  const uint4* src = reinterpret_cast<const uint4*>(d_table);
  uint4* dst = reinterpret_cast<uint4*>(sm->table);
  // the walk masks every next-node field to 8 bits, so any table stays in range
  for (int i = threadIdx.x; i < 256 * 16 / 2; i += kThreads) dst[i] = __ldg(src + i);
  for (int z = threadIdx.x; z <= kPadBits; z += kThreads) sm->zero_codes[z] = (uint16_t)(z / a.lmin);
  __syncthreads();
  const uint32_t warp = threadIdx.x >> 5;
  uint32_t g = blockIdx.x * kWarps + warp;
  if (g >= a.n_groups) return;
  GroupIn in;
  fetch_group(a, g, in);
  for (; g < a.n_groups; g += gridDim.x * kWarps) {
    GroupIn nx;
    const uint32_t gn = g + gridDim.x * kWarps;
    const bool more = gn < a.n_groups;
    if (more) fetch_group(a, gn, nx);
    process_group(a, g, in, sm, &sm->warp[warp], status);
    if (more) in = nx;
  }
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

}  // namespace
}  // namespace ecf8_bf16

using namespace ecf8_bf16;

extern "C" int ecf8_bf16_decode(const ecf8_bf16_info* info, const void* d_blob, const void* d_table, uint16_t* d_out,
                                size_t n, int32_t* d_status, cudaStream_t s) {
  if (!info || n != info->n) return ECF8_ERR_ARG;
  if (info->chunk_bytes != (uint32_t)kC || info->group_chunks != (uint32_t)kT) return ECF8_ERR_UNSUPPORTED;
  if (n == 0) return ECF8_OK;
  if (!d_blob || !d_table || !d_out) return ECF8_ERR_ARG;
  if (!aligned16(d_blob) || !aligned16(d_table) || !aligned16(d_out)) return ECF8_ERR_ALIGN;
  uint32_t lmin = 16;
  for (int v = 0; v < 256; ++v)
    if (info->len[v] && info->len[v] < lmin) lmin = info->len[v];
  const uint8_t* b = static_cast<const uint8_t*>(d_blob);
  Args a;
  a.gaps = reinterpret_cast<const uint32_t*>(b + info->gaps_off);
  a.groups = reinterpret_cast<const uint64_t*>(b + info->groups_off);
  a.stream = reinterpret_cast<const uint32_t*>(b + info->stream_off);
  a.kept = b + info->kept_off;
  a.out = d_out;
  a.n = info->n;
  a.code_bits = info->code_bits;
  a.n_groups = info->n_groups;
  a.lmin = lmin;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev))
    return ECF8_ERR_CUDA;
  if (cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Smem)))
    return ECF8_ERR_CUDA;
  const uint64_t ctas_needed = ((uint64_t)a.n_groups + kWarps - 1) / kWarps;
  const uint32_t grid = (uint32_t)(ctas_needed < (uint64_t)sms ? ctas_needed : (uint64_t)sms);
  decode_kernel<<<grid, kThreads, sizeof(Smem), s>>>(static_cast<const uint2*>(d_table), a, d_status);
  if (cudaGetLastError() != cudaSuccess) return ECF8_ERR_CUDA;
  ecf8::note_launch();
  return ECF8_OK;
}
