// ECF8 GPU decoder for sm_100a.
//
// Reconstructs FP8 E4M3 bytes from a Huffman-coded exponent stream and a
// sign/mantissa nibble array (ECF8 walkthrough "ECF8 浮点数压缩技术" §3.2.1, the
// decode_kernel pipeline; arXiv 2510.02676 abstract).  The pages' kernel is
// prior art written for H100/RTX40 parts; this one keeps its idea -- every
// thread owns a fixed slice of the bit stream, starts at a stored gap, counts
// its codes, and a block-wide prefix sum of the counts places its output --
// and is otherwise laid out for B200:
//
//  * one CTA of T threads decodes one group of T chunks (C bytes of stream
//    each); the group's first output index comes from the stored offsets, so
//    CTAs never wait on each other;
//  * each thread walks its chunk ONCE with a 4096-entry table in shared
//    memory that yields up to six codes per lookup, and parks the exponents
//    (4 bits each) in a thread-private, bank-interleaved smem area;
//  * a warp-shuffle scan (plus one smem step across warps) of the per-thread
//    code counts gives every thread its output position; threads then
//    funnel-shift their exponents into one contiguous, 32-weight-aligned
//    staging array;
//  * the CTA finally streams its output range in 32-weight blocks: 16 bytes
//    of staged exponents + one 16-byte nibble load -> 32 output bytes with
//    byte-permute and 3-input logic ops, stored as two 16-byte vectors.
//
// The path is HBM-bound integer work: no tensor cores.  Corrupt input is
// reported through a status word; no access leaves its buffer and no loop
// runs without a bound.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <vector>

#include "ecf8.h"
#include "ecf8_format.h"

namespace ecf8 {
namespace {

constexpr int kK = (int)kLutBits;

template <int C, int T>
struct Shape {
  static_assert(C % 16 == 0 && T % 32 == 0 && T <= 1024, "unsupported layout");
  static constexpr int kWords = C / 4;          // stream words per chunk
  static constexpr int kPrivWords = C;          // 8C codes of 4 bits at most
  static constexpr int kMaxCodes = 8 * C * T;   // per group
  static constexpr int kStageWords = T * C + 8; // staged exponents, +32 for alignment
  static constexpr int kWarps = T / 32;
  // shared memory carve-up, in 32-bit words
  static constexpr int kLutOff = 0;
  static constexpr int kPrivOff = kLutOff + (int)kLutEntries;
  static constexpr int kStageOff = kPrivOff + kPrivWords * T;
  static constexpr int kScanOff = kStageOff + kStageWords;
  static constexpr int kCanonOff = kScanOff + 72;  // warp sums, exclusive prefixes, total
  static constexpr int kCanonWords = 17 * 3 + 4 + 4;  // first, count, base; sorted[16]; len[16]
  static constexpr size_t kSmemBytes = 4ull * (kCanonOff + kCanonWords);
};

// Canonical decoding tables for codes longer than the 12-bit window (rare).
struct Canon {
  uint32_t first[17];
  uint32_t count[17];
  uint32_t base[17];
  uint8_t sorted[16];
  uint8_t len[16];
};

__device__ __forceinline__ void build_canon(const uint8_t* len, Canon* c) {
  uint32_t cnt[17] = {};
  for (int s = 0; s < 16; ++s) cnt[len[s]]++;
  cnt[0] = 0;
  uint32_t code = 0, base = 0;
  for (int l = 1; l <= 16; ++l) {
    code = (code + cnt[l - 1]) << 1;
    c->first[l] = code;
    c->count[l] = cnt[l];
    c->base[l] = base;
    base += cnt[l];
  }
  c->first[0] = c->count[0] = c->base[0] = 0;
  uint32_t k = 0;
  for (int l = 1; l <= 16; ++l)
    for (int s = 0; s < 16; ++s)
      if (len[s] == l) c->sorted[k++] = (uint8_t)s;
  for (int s = 0; s < 16; ++s) c->len[s] = len[s];
}

// bitselect: bits of a where m is set, bits of b elsewhere (one LOP3)
__device__ __forceinline__ uint32_t bsel(uint32_t m, uint32_t a, uint32_t b) { return (a & m) | (b & ~m); }

// 8 weights: E = their exponents, 4 bits each in order; N = their nibble
// word (weight k<4 in byte k low half, weight 4+k in byte k high half).
__device__ __forceinline__ void assemble8(uint32_t E, uint32_t N, uint32_t& lo, uint32_t& hi) {
  const uint32_t n_lo = bsel(0x80808080u, N << 4, N);  // sign to bit 7, mantissa in bits 0-2
  const uint32_t n_hi = bsel(0x80808080u, N, N >> 4);
  const uint32_t x_lo = __byte_perm(E, 0, 0x1100);     // bytes e1e0 e1e0 e3e2 e3e2
  const uint32_t x_hi = __byte_perm(E, 0, 0x3322);
  const uint32_t e_lo = bsel(0x00FF00FFu, x_lo << 3, x_lo >> 1);  // even bytes low nibble, odd high
  const uint32_t e_hi = bsel(0x00FF00FFu, x_hi << 3, x_hi >> 1);
  lo = bsel(0x78787878u, e_lo, n_lo);
  hi = bsel(0x78787878u, e_hi, n_hi);
}

struct Walker {
  uint64_t buf;  // next stream bits, MSB-aligned
  int valid;     // bits of buf that are stream bits
  int pos;       // chunk-relative bit of the next code start
  int end;       // decode codes starting before this bit
  uint64_t acc;  // exponents not yet parked, 4 bits each, first in the low bits
  int nacc;
  int nw;        // words parked
  bool bad;
};

template <int C, int T>
__device__ __forceinline__ void park(Walker& w, uint32_t* priv, uint32_t syms, int cnt) {
  using S = Shape<C, T>;
  w.acc |= (uint64_t)syms << (4 * w.nacc);
  w.nacc += cnt;
  if (w.nacc >= 8) {
    priv[min(w.nw, S::kPrivWords - 1) * T + threadIdx.x] = (uint32_t)w.acc;
    w.nw++;
    w.acc >>= 32;
    w.nacc -= 8;
  }
}

// One code by canonical decoding of a 16-bit window; false on bits that
// match no code (a corrupt stream, or a one-code book seeing a 1).
__device__ __forceinline__ bool canon_one(const Canon* c, uint64_t buf, uint32_t& sym, int& len) {
  const uint32_t win = (uint32_t)(buf >> 48);
#pragma unroll 1
  for (int l = 1; l <= 16; ++l) {
    const uint32_t v = (win >> (16 - l)) - c->first[l];
    if (v < c->count[l]) {
      sym = c->sorted[c->base[l] + v];
      len = l;
      return true;
    }
  }
  return false;
}

template <int C, int T>
__device__ __forceinline__ void step_multi(Walker& w, const uint32_t* lut, const Canon* canon, uint32_t* priv) {
  const uint32_t e = lut[(uint32_t)(w.buf >> (64 - kK))];
  const int cnt = (e >> 4) & 7, nb = e & 15;
  if (cnt != 0 && nb != 0) {
    park<C, T>(w, priv, e >> 8, cnt);
    w.buf <<= nb;
    w.valid -= nb;
    w.pos += nb;
    return;
  }
  uint32_t sym;
  int len;
  if (!canon_one(canon, w.buf, sym, len)) {
    w.bad = true;
    w.end = w.pos;  // stop this thread
    return;
  }
  park<C, T>(w, priv, sym, 1);
  w.buf <<= len;
  w.valid -= len;
  w.pos += len;
}

template <int C, int T>
__device__ __forceinline__ void step_single(Walker& w, const uint32_t* lut, const Canon* canon, uint32_t* priv) {
  const uint32_t e = lut[(uint32_t)(w.buf >> (64 - kK))];
  uint32_t sym = (e >> 8) & 15;
  int len = canon->len[sym];
  if (((e >> 4) & 7) == 0 || len == 0) {
    if (!canon_one(canon, w.buf, sym, len)) {
      w.bad = true;
      w.end = w.pos;
      return;
    }
  }
  park<C, T>(w, priv, sym, 1);
  w.buf <<= len;
  w.valid -= len;
  w.pos += len;
}

template <int C, int T>
__device__ __forceinline__ void decode_group(const DevTensor& d, uint32_t g, uint32_t* sm, int32_t* status) {
  using S = Shape<C, T>;
  uint32_t* lut = sm + S::kLutOff;
  uint32_t* priv = sm + S::kPrivOff;
  uint32_t* stage = sm + S::kStageOff;
  uint32_t* scan = sm + S::kScanOff;
  Canon* canon = reinterpret_cast<Canon*>(sm + S::kCanonOff);
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;

  // K0: decode table and canonical tables into shared memory
  {
    const uint4* src = reinterpret_cast<const uint4*>(d.lut);
    uint4* dst = reinterpret_cast<uint4*>(lut);
#pragma unroll 4
    for (int i = t; i < (int)kLutEntries / 4; i += T) dst[i] = __ldg(src + i);
    if (t == 0) build_canon(d.len, canon);
  }
  const uint64_t off0 = __ldg(d.groups + g), off1 = __ldg(d.groups + g + 1);

  // K1: this thread's chunk (+ the next word for a code that straddles the end)
  const uint64_t chunk = (uint64_t)g * T + t;
  const uint64_t bit0 = chunk * (8ull * C);
  Walker w;
  const uint64_t left = bit0 < d.code_bits ? d.code_bits - bit0 : 0;
  w.end = left < 8ull * C ? (int)left : 8 * C;
  const uint32_t gap = (__ldg(d.gaps + (chunk >> 3)) >> ((chunk & 7) * 4)) & 15u;
  uint32_t word[S::kWords + 1];
  {
    const uint4* cs = reinterpret_cast<const uint4*>(d.stream + chunk * S::kWords);
#pragma unroll
    for (int q = 0; q < S::kWords / 4; ++q) {
      const uint4 v = __ldg(cs + q);
      word[4 * q + 0] = v.x;
      word[4 * q + 1] = v.y;
      word[4 * q + 2] = v.z;
      word[4 * q + 3] = v.w;
    }
    word[S::kWords] = __ldg(d.stream + (chunk + 1) * S::kWords);
  }
  w.buf = (((uint64_t)word[0] << 32) | word[1]) << gap;
  w.valid = 64 - (int)gap;
  w.pos = (int)gap;
  w.acc = 0;
  w.nacc = 0;
  w.nw = 0;
  w.bad = false;
  __syncthreads();  // tables ready

  // K2: walk the chunk once.  Full-window lookups while every code the entry
  // holds is sure to start before `end`, then one code at a time.
#pragma unroll
  for (int k = 2; k <= S::kWords; ++k) {
    while (w.valid > 32 && w.pos + kK <= w.end) step_multi<C, T>(w, lut, canon, priv);
    if (w.valid > 32) break;  // at the tail with >= 20 bits buffered past `end`
    w.buf |= (uint64_t)word[k] << (32 - w.valid);
    w.valid += 32;
  }
  while (w.pos + kK <= w.end) step_multi<C, T>(w, lut, canon, priv);
  while (w.pos < w.end) step_single<C, T>(w, lut, canon, priv);
  if (w.nacc > 0) priv[min(w.nw, S::kPrivWords - 1) * T + t] = (uint32_t)w.acc;
  const uint32_t cnt = (uint32_t)(w.nw * 8 + w.nacc);
  const bool overflow = w.nw > S::kPrivWords || (w.nw == S::kPrivWords && w.nacc > 0);

  // K3: place -- warp-shuffle inclusive scan, then across warps
  uint32_t incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) scan[warp] = incl;
  const int any_bad = __syncthreads_or(w.bad || overflow);
  if (warp == 0) {
    const uint32_t v = lane < S::kWarps ? scan[lane] : 0;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
      if (lane >= o) x += y;
    }
    if (lane < S::kWarps) scan[32 + lane] = x - v;
    if (lane == S::kWarps - 1) scan[64] = x;
  }
  __syncthreads();
  const uint32_t total = scan[64];
  const uint32_t start = incl - cnt + scan[32 + warp];

  const bool offsets_ok = off0 <= off1 && off1 <= d.n && off1 - off0 <= (uint64_t)S::kMaxCodes;
  if (any_bad || !offsets_ok || (uint64_t)total != off1 - off0) {
    if (t == 0 && status) {
      int32_t f = 0;
      if (any_bad) f |= ECF8_STATUS_BAD_CODE;
      if (!offsets_ok) f |= ECF8_STATUS_BAD_OFFSETS;
      else if ((uint64_t)total != off1 - off0) f |= ECF8_STATUS_COUNT_MISMATCH;
      atomicOr(status, f);
    }
    return;  // uniform across the CTA
  }

  // K4a: funnel-shift this thread's exponents to stage[] nibble position
  // (off0 mod 32) + start, so that stage word 4b.. covers output block b
  const uint32_t q = (uint32_t)(off0 & 31) + start;
  const uint32_t d0 = q >> 3, dl = cnt ? (q + cnt - 1) >> 3 : 0;
  if (cnt) {
    stage[d0] = 0;
    stage[dl] = 0;
  }
  __syncthreads();
  if (cnt) {
    const uint32_t r = (q & 7) * 4;
    const uint32_t used = (cnt + 7) / 8;
    uint32_t prev = 0;
    for (uint32_t j = 0; j <= dl - d0; ++j) {
      const uint32_t cur = j < used ? priv[j * T + t] : 0;
      const uint32_t v = __funnelshift_l(prev, cur, r);
      prev = cur;
      if (j == 0 || j == dl - d0)
        atomicOr(&stage[d0 + j], v);
      else
        stage[d0 + j] = v;
    }
  }
  __syncthreads();

  // K4b + K5: assemble 32 weights per step and store them
  const uint64_t base = off0 & ~31ull;
  const uint32_t blocks = ((uint32_t)(off0 & 31) + total + 31) >> 5;
  const uint4* nib = reinterpret_cast<const uint4*>(d.nibbles);
  for (uint32_t b = t; b < blocks; b += T) {
    const uint4 ex = reinterpret_cast<const uint4*>(stage)[b];
    const uint64_t gpos = base + 32ull * b;
    const uint4 nb = __ldg(nib + (gpos >> 5));
    uint32_t o[8];
    assemble8(ex.x, nb.x, o[0], o[1]);
    assemble8(ex.y, nb.y, o[2], o[3]);
    assemble8(ex.z, nb.z, o[4], o[5]);
    assemble8(ex.w, nb.w, o[6], o[7]);
    const uint64_t lo = gpos > off0 ? gpos : off0;
    const uint64_t hi = gpos + 32 < off1 ? gpos + 32 : off1;
    uint8_t* dst = d.out + gpos;
    if (lo == gpos && hi == gpos + 32) {
      reinterpret_cast<uint4*>(dst)[0] = make_uint4(o[0], o[1], o[2], o[3]);
      reinterpret_cast<uint4*>(dst)[1] = make_uint4(o[4], o[5], o[6], o[7]);
    } else {
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const uint64_t i = gpos + k;
        if (i >= lo && i < hi) dst[k] = (uint8_t)(o[k >> 2] >> (8 * (k & 3)));
      }
    }
  }
}

template <int C, int T>
__global__ void __launch_bounds__(T) decode_one_kernel(const DevTensor d, int32_t* status) {
  extern __shared__ __align__(16) uint32_t smem[];
  decode_group<C, T>(d, blockIdx.x, smem, status);
}

// the tensor whose groups contain group g: the last with group_base <= g
__device__ __forceinline__ int find_tensor(const DevTensor* ts, int count, uint32_t g) {
  int lo = 0, hi = count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ts[mid].group_base <= g) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

template <int C, int T>
__global__ void __launch_bounds__(T) decode_many_kernel(const DevTensor* __restrict__ ts, int count, int32_t* status) {
  extern __shared__ __align__(16) uint32_t smem[];
  const DevTensor d = ts[find_tensor(ts, count, blockIdx.x)];
  decode_group<C, T>(d, blockIdx.x - d.group_base, smem, status);
}

// Small batches travel inside the launch's parameter block.
constexpr int kInlineMax = ECF8_BATCH_INLINE_MAX;
struct InlineBatch {
  DevTensor t[kInlineMax];
  int count;
};

template <int C, int T>
__global__ void __launch_bounds__(T) decode_inline_kernel(const __grid_constant__ InlineBatch b, int32_t* status) {
  extern __shared__ __align__(16) uint32_t smem[];
  const DevTensor d = b.t[find_tensor(b.t, b.count, blockIdx.x)];
  decode_group<C, T>(d, blockIdx.x - d.group_base, smem, status);
}

std::atomic<uint64_t> g_launches{0};

template <int C, int T>
int set_smem_attr() {
  // per device, once
  static std::atomic<uint64_t> done_mask{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ECF8_ERR_CUDA;
  const uint64_t bit = 1ull << (dev & 63);
  if (done_mask.load() & bit) return ECF8_OK;
  using S = Shape<C, T>;
  if (cudaFuncSetAttribute(decode_one_kernel<C, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)S::kSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(decode_many_kernel<C, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)S::kSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(decode_inline_kernel<C, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)S::kSmemBytes) != cudaSuccess)
    return ECF8_ERR_CUDA;
  done_mask.fetch_or(bit);
  return ECF8_OK;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

int check_info(const ecf8_info* info) {
  if (!info) return ECF8_ERR_ARG;
  if (info->lut_bits != kLutBits) return ECF8_ERR_UNSUPPORTED;
  Layout L;
  if (!compute_layout(info->n, info->code_bits, info->chunk_bytes, info->group_chunks, &L)) return ECF8_ERR_FORMAT;
  if (L.groups != info->n_groups || L.total != info->blob_bytes || L.lut_off != info->lut_off ||
      L.gaps_off != info->gaps_off || L.groups_off != info->groups_off || L.stream_off != info->stream_off ||
      L.nib_off != info->nibbles_off)
    return ECF8_ERR_FORMAT;
  // the kernels index their canonical tables by code length: lengths must be
  // a prefix code of at most 16 bits
  uint64_t kraft = 0;
  for (int s = 0; s < 16; ++s) {
    if (info->len[s] > 16) return ECF8_ERR_CODEBOOK;
    if (info->len[s]) kraft += 1ull << (16 - info->len[s]);
  }
  if (kraft > (1ull << 16) || (info->n && kraft == 0)) return ECF8_ERR_CODEBOOK;
  return ECF8_OK;
}

DevTensor make_dev(const ecf8_info* info, const void* d_blob, uint8_t* d_out) {
  const uint8_t* b = static_cast<const uint8_t*>(d_blob);
  DevTensor t;
  t.lut = reinterpret_cast<const uint32_t*>(b + info->lut_off);
  t.gaps = reinterpret_cast<const uint32_t*>(b + info->gaps_off);
  t.groups = reinterpret_cast<const uint64_t*>(b + info->groups_off);
  t.stream = reinterpret_cast<const uint32_t*>(b + info->stream_off);
  t.nibbles = b + info->nibbles_off;
  t.out = d_out;
  t.n = info->n;
  t.code_bits = info->code_bits;
  t.n_groups = info->n_groups;
  t.group_base = 0;
  for (int s = 0; s < 16; ++s) t.len[s] = info->len[s];
  return t;
}

constexpr int kC = 32, kT = 128;  // the layout the kernels are built for

}  // namespace
}  // namespace ecf8

using namespace ecf8;

extern "C" {

int ecf8_layout_supported(uint32_t chunk_bytes, uint32_t group_chunks) {
  return chunk_bytes == (uint32_t)kC && group_chunks == (uint32_t)kT;
}

int ecf8_decode(const ecf8_info* info, const void* d_blob, uint8_t* d_out, size_t n, int32_t* d_status,
                cudaStream_t s) {
  int rc = check_info(info);
  if (rc) return rc;
  if (n != info->n) return ECF8_ERR_ARG;
  if (n == 0) return ECF8_OK;
  if (!d_blob || !d_out) return ECF8_ERR_ARG;
  if (!aligned16(d_blob) || !aligned16(d_out)) return ECF8_ERR_ALIGN;
  if (!ecf8_layout_supported(info->chunk_bytes, info->group_chunks)) return ECF8_ERR_UNSUPPORTED;
  if ((rc = set_smem_attr<kC, kT>())) return rc;
  const DevTensor t = make_dev(info, d_blob, d_out);
  decode_one_kernel<kC, kT><<<info->n_groups, kT, Shape<kC, kT>::kSmemBytes, s>>>(t, d_status);
  if (cudaGetLastError() != cudaSuccess) return ECF8_ERR_CUDA;
  g_launches.fetch_add(1);
  return ECF8_OK;
}

size_t ecf8_batched_workspace_size(int count) {
  return count > kInlineMax ? sizeof(DevTensor) * (size_t)count : 0;
}

int ecf8_decode_batched(const ecf8_tensor* tensors, int count, void* d_workspace, size_t workspace_bytes,
                        int32_t* d_status, cudaStream_t s) {
  if (count < 0 || (count > 0 && !tensors)) return ECF8_ERR_ARG;
  if (count == 0) return ECF8_OK;
  if (count > kInlineMax) {
    if (!d_workspace || workspace_bytes < ecf8_batched_workspace_size(count)) return ECF8_ERR_WORKSPACE;
    if (!aligned16(d_workspace)) return ECF8_ERR_ALIGN;
  }
  std::vector<DevTensor> host;
  host.reserve(count);
  uint64_t groups = 0;
  for (int i = 0; i < count; ++i) {
    const ecf8_tensor& x = tensors[i];
    int rc = check_info(x.info);
    if (rc) return rc;
    if (!ecf8_layout_supported(x.info->chunk_bytes, x.info->group_chunks)) return ECF8_ERR_UNSUPPORTED;
    if (x.info->n == 0) continue;
    if (!x.d_blob || !x.d_out) return ECF8_ERR_ARG;
    if (!aligned16(x.d_blob) || !aligned16(x.d_out)) return ECF8_ERR_ALIGN;
    DevTensor t = make_dev(x.info, x.d_blob, x.d_out);
    t.group_base = (uint32_t)groups;
    groups += x.info->n_groups;
    if (groups > 0x7FFFFFFFull) return ECF8_ERR_UNSUPPORTED;
    host.push_back(t);
  }
  if (host.empty()) return ECF8_OK;
  int rc = set_smem_attr<kC, kT>();
  if (rc) return rc;
  if (host.size() <= (size_t)kInlineMax) {
    InlineBatch b;
    for (size_t i = 0; i < host.size(); ++i) b.t[i] = host[i];
    b.count = (int)host.size();
    decode_inline_kernel<kC, kT><<<(unsigned)groups, kT, Shape<kC, kT>::kSmemBytes, s>>>(b, d_status);
  } else {
    if (cudaMemcpyAsync(d_workspace, host.data(), sizeof(DevTensor) * host.size(), cudaMemcpyHostToDevice, s) !=
        cudaSuccess)
      return ECF8_ERR_CUDA;
    decode_many_kernel<kC, kT><<<(unsigned)groups, kT, Shape<kC, kT>::kSmemBytes, s>>>(
        static_cast<const DevTensor*>(d_workspace), (int)host.size(), d_status);
  }
  if (cudaGetLastError() != cudaSuccess) return ECF8_ERR_CUDA;
  g_launches.fetch_add(1);
  return ECF8_OK;
}

uint64_t ecf8_launch_count(void) { return g_launches.load(); }

}  // extern "C"
