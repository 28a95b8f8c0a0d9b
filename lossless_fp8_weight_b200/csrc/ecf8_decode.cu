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
#include <mutex>
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
  static constexpr int kNB = 8;          // nibble blocks a thread prefetches in registers
  static constexpr int kMinBlocks = 4;   // CTAs per SM the smem budget allows
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

// ---------------------------------------------------------------- per group

// What one thread fetches ahead for a group: its stream slice (+ the next
// word, for a code that straddles the slice end), the raw gap word, and the
// group's two offsets.  Kept raw so the loads stay in flight until used.
template <int C>
struct GroupIn {
  uint32_t w[C / 4 + 1];
  uint32_t gapw;
  uint64_t off0, off1;
};

template <int C, int T>
__device__ __forceinline__ void fetch_group(const DevTensor* dt, uint32_t local, GroupIn<C>& in) {
  using S = Shape<C, T>;
  const uint64_t chunk = (uint64_t)local * T + threadIdx.x;
  const uint32_t* stream = dt->stream;
  const uint4* cs = reinterpret_cast<const uint4*>(stream + chunk * S::kWords);
#pragma unroll
  for (int q = 0; q < S::kWords / 4; ++q) {
    const uint4 v = __ldg(cs + q);
    in.w[4 * q + 0] = v.x;
    in.w[4 * q + 1] = v.y;
    in.w[4 * q + 2] = v.z;
    in.w[4 * q + 3] = v.w;
  }
  in.w[S::kWords] = __ldg(stream + (chunk + 1) * S::kWords);
  in.gapw = __ldg(dt->gaps + (chunk >> 3));
  in.off0 = __ldg(dt->groups + local);
  in.off1 = __ldg(dt->groups + local + 1);
}

// K0: the tensor's decode table and canonical tables into shared memory.
template <int C, int T>
__device__ __forceinline__ void load_tables(const DevTensor* dt, uint32_t* lut, Canon* canon) {
  const uint4* src = reinterpret_cast<const uint4*>(dt->lut);
  uint4* dst = reinterpret_cast<uint4*>(lut);
#pragma unroll 4
  for (int i = threadIdx.x; i < (int)kLutEntries / 4; i += T) dst[i] = __ldg(src + i);
  if (threadIdx.x == 0) build_canon(dt->len, canon);
  __syncthreads();
}

// K4b + K5 for one 32-weight block: staged exponents + nibbles -> 32 bytes.
__device__ __forceinline__ void store_block(uint8_t* out, uint64_t gpos, uint64_t off0, uint64_t off1, const uint4 ex,
                                            const uint4 nb) {
  uint32_t o[8];
  assemble8(ex.x, nb.x, o[0], o[1]);
  assemble8(ex.y, nb.y, o[2], o[3]);
  assemble8(ex.z, nb.z, o[4], o[5]);
  assemble8(ex.w, nb.w, o[6], o[7]);
  uint8_t* dst = out + gpos;
  if (gpos >= off0 && gpos + 32 <= off1) {
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(o[0], o[1], o[2], o[3]);
    reinterpret_cast<uint4*>(dst)[1] = make_uint4(o[4], o[5], o[6], o[7]);
  } else {  // the group's ragged ends: bytes inside [off0, off1) only
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const uint64_t i = gpos + k;
      if (i >= off0 && i < off1) dst[k] = (uint8_t)(o[k >> 2] >> (8 * (k & 3)));
    }
  }
}

template <int C, int T>
__device__ __forceinline__ void process_group(const DevTensor* dt, uint32_t local, const GroupIn<C>& in, uint32_t* sm,
                                              int32_t* status) {
  using S = Shape<C, T>;
  uint32_t* lut = sm + S::kLutOff;
  uint32_t* priv = sm + S::kPrivOff;
  uint32_t* stage = sm + S::kStageOff;
  uint32_t* scan = sm + S::kScanOff;
  const Canon* canon = reinterpret_cast<const Canon*>(sm + S::kCanonOff);
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const uint64_t n = dt->n;
  const uint64_t off0 = in.off0, off1 = in.off1;
  const bool offsets_ok = off0 <= off1 && off1 <= n && off1 - off0 <= (uint64_t)S::kMaxCodes;

  // this group's nibbles: issued now, consumed after the walk
  const uint32_t blocks = offsets_ok ? (uint32_t)(((off0 & 31) + (off1 - off0) + 31) >> 5) : 0;
  const uint4* nib = reinterpret_cast<const uint4*>(dt->nibbles) + (off0 >> 5);
  uint4 nv[S::kNB];
#pragma unroll
  for (int j = 0; j < S::kNB; ++j)
    if ((uint32_t)(t + j * T) < blocks) nv[j] = __ldg(nib + t + j * T);

  // K2: walk the chunk once.  Full-window lookups while every code the entry
  // holds is sure to start before `end`, then one code at a time.
  const uint64_t bit0 = ((uint64_t)local * T + t) * (8ull * C);
  const uint64_t code_bits = dt->code_bits;
  const uint64_t left = bit0 < code_bits ? code_bits - bit0 : 0;
  const uint32_t gap = (in.gapw >> ((t & 7) * 4)) & 15u;
  Walker w;
  w.end = left < 8ull * C ? (int)left : 8 * C;
  w.buf = (((uint64_t)in.w[0] << 32) | in.w[1]) << gap;
  w.valid = 64 - (int)gap;
  w.pos = (int)gap;
  w.acc = 0;
  w.nacc = 0;
  w.nw = 0;
  w.bad = false;
#pragma unroll
  for (int k = 2; k <= S::kWords; ++k) {
    while (w.valid > 32 && w.pos + kK <= w.end) step_multi<C, T>(w, lut, canon, priv);
    if (w.valid > 32) break;  // at the tail with >= 20 bits buffered past `end`
    w.buf |= (uint64_t)in.w[k] << (32 - w.valid);
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
  // (off0 mod 32) + start, so that stage words 4b..4b+3 cover output block b
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

  // K4b + K5
  const uint64_t base = off0 & ~31ull;
  const uint4* st = reinterpret_cast<const uint4*>(stage);
  uint8_t* out = dt->out;
#pragma unroll
  for (int j = 0; j < S::kNB; ++j) {
    const uint32_t b = t + j * T;
    if (b < blocks) store_block(out, base + 32ull * b, off0, off1, st[b], nv[j]);
  }
  for (uint32_t b = t + S::kNB * T; b < blocks; b += T) store_block(out, base + 32ull * b, off0, off1, st[b], __ldg(nib + b));
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

// Persistent CTA: a contiguous run of groups (across tensors, in table order).
// The next group's stream slice and offsets are fetched while this one is
// decoded; the decode table is reloaded only when the run enters a new tensor.
template <int C, int T>
__device__ __forceinline__ void decode_run(const DevTensor* table, int count, uint32_t total, int32_t* status) {
  using S = Shape<C, T>;
  extern __shared__ __align__(16) uint32_t smem[];
  const uint32_t gb = (uint32_t)((uint64_t)blockIdx.x * total / gridDim.x);
  const uint32_t ge = (uint32_t)((uint64_t)(blockIdx.x + 1) * total / gridDim.x);
  if (gb >= ge) return;
  int ti = find_tensor(table, count, gb);
  load_tables<C, T>(table + ti, smem + S::kLutOff, reinterpret_cast<Canon*>(smem + S::kCanonOff));
  GroupIn<C> in;
  fetch_group<C, T>(table + ti, gb - table[ti].group_base, in);
  for (uint32_t g = gb; g < ge; ++g) {
    const DevTensor* dt = table + ti;
    const uint32_t base = dt->group_base;
    const bool more = g + 1 < ge;
    const bool next_tensor = more && g + 1 >= base + dt->n_groups;
    GroupIn<C> nx;
    if (more) fetch_group<C, T>(dt + (next_tensor ? 1 : 0), g + 1 - (next_tensor ? dt[1].group_base : base), nx);
    process_group<C, T>(dt, g - base, in, smem, status);
    if (more) {
      if (next_tensor) {  // every thread is past the walk of group g
        ++ti;
        load_tables<C, T>(table + ti, smem + S::kLutOff, reinterpret_cast<Canon*>(smem + S::kCanonOff));
      }
      in = nx;
    }
  }
}

template <int C, int T>
__global__ void __launch_bounds__(T, Shape<C, T>::kMinBlocks) decode_table_kernel(const DevTensor* __restrict__ ts,
                                                                                    int count, uint32_t total,
                                                                                    int32_t* status) {
  decode_run<C, T>(ts, count, total, status);
}

// Small batches travel inside the launch's parameter block.
template <int N>
struct InlineBatch {
  DevTensor t[N];
  int count;
};
constexpr int kInlineMax = ECF8_BATCH_INLINE_MAX;

template <int C, int T, int N>
__global__ void __launch_bounds__(T, Shape<C, T>::kMinBlocks) decode_inline_kernel(
    const __grid_constant__ InlineBatch<N> b, uint32_t total, int32_t* status) {
  decode_run<C, T>(b.t, b.count, total, status);
}

std::atomic<uint64_t> g_launches{0};

// Per device, once: allow the kernels their shared memory and size the
// persistent grid (resident CTAs per SM x SMs).
template <int C, int T>
int grid_for_device(uint32_t* ctas) {
  struct Entry {
    std::atomic<uint32_t> ctas{0};
  };
  static Entry per_dev[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ECF8_ERR_CUDA;
  uint32_t have = per_dev[dev].ctas.load();
  if (have) {
    *ctas = have;
    return ECF8_OK;
  }
  using S = Shape<C, T>;
  const int bytes = (int)S::kSmemBytes;
  if (cudaFuncSetAttribute(decode_table_kernel<C, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ||
      cudaFuncSetAttribute(decode_inline_kernel<C, T, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ||
      cudaFuncSetAttribute(decode_inline_kernel<C, T, kInlineMax>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           bytes))
    return ECF8_ERR_CUDA;
  int sms = 0, per_sm = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_inline_kernel<C, T, kInlineMax>, T, bytes))
    return ECF8_ERR_CUDA;
  have = (uint32_t)(sms * (per_sm > 0 ? per_sm : 1));
  per_dev[dev].ctas.store(have);
  *ctas = have;
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

// Checks one tensor of a call and appends its descriptor (skipping n = 0).
int add_tensor(const ecf8_info* info, const void* d_blob, uint8_t* d_out, std::vector<DevTensor>& v,
               uint64_t& groups) {
  int rc = check_info(info);
  if (rc) return rc;
  if (info->chunk_bytes != (uint32_t)kC || info->group_chunks != (uint32_t)kT) return ECF8_ERR_UNSUPPORTED;
  if (info->n == 0) return ECF8_OK;
  if (!d_blob || !d_out) return ECF8_ERR_ARG;
  if (!aligned16(d_blob) || !aligned16(d_out)) return ECF8_ERR_ALIGN;
  DevTensor t = make_dev(info, d_blob, d_out);
  t.group_base = (uint32_t)groups;
  groups += info->n_groups;
  if (groups > 0xFFFFFFFFull) return ECF8_ERR_UNSUPPORTED;
  v.push_back(t);
  return ECF8_OK;
}

uint32_t grid_size(uint32_t ctas, uint64_t groups) { return (uint32_t)(groups < ctas ? groups : ctas); }

}  // namespace
}  // namespace ecf8

using namespace ecf8;

extern "C" {

int ecf8_layout_supported(uint32_t chunk_bytes, uint32_t group_chunks) {
  return chunk_bytes == (uint32_t)kC && group_chunks == (uint32_t)kT;
}

int ecf8_decode(const ecf8_info* info, const void* d_blob, uint8_t* d_out, size_t n, int32_t* d_status,
                cudaStream_t s) {
  if (!info) return ECF8_ERR_ARG;
  if (n != info->n) return ECF8_ERR_ARG;
  std::vector<DevTensor> v;
  uint64_t groups = 0;
  int rc = add_tensor(info, d_blob, d_out, v, groups);
  if (rc || v.empty()) return rc;
  uint32_t ctas = 0;
  if ((rc = grid_for_device<kC, kT>(&ctas))) return rc;
  InlineBatch<1> b;
  b.t[0] = v[0];
  b.count = 1;
  decode_inline_kernel<kC, kT, 1><<<grid_size(ctas, groups), kT, Shape<kC, kT>::kSmemBytes, s>>>(
      b, (uint32_t)groups, d_status);
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
  std::vector<DevTensor> v;
  v.reserve(count);
  uint64_t groups = 0;
  for (int i = 0; i < count; ++i) {
    int rc = add_tensor(tensors[i].info, tensors[i].d_blob, tensors[i].d_out, v, groups);
    if (rc) return rc;
  }
  if (v.empty()) return ECF8_OK;
  uint32_t ctas = 0;
  int rc = grid_for_device<kC, kT>(&ctas);
  if (rc) return rc;
  const uint32_t grid = grid_size(ctas, groups);
  if (v.size() <= (size_t)kInlineMax) {
    InlineBatch<kInlineMax> b;
    for (size_t i = 0; i < v.size(); ++i) b.t[i] = v[i];
    b.count = (int)v.size();
    decode_inline_kernel<kC, kT, kInlineMax><<<grid, kT, Shape<kC, kT>::kSmemBytes, s>>>(b, (uint32_t)groups,
                                                                                          d_status);
  } else {
    if (cudaMemcpyAsync(d_workspace, v.data(), sizeof(DevTensor) * v.size(), cudaMemcpyHostToDevice, s) !=
        cudaSuccess)
      return ECF8_ERR_CUDA;
    decode_table_kernel<kC, kT><<<grid, kT, Shape<kC, kT>::kSmemBytes, s>>>(
        static_cast<const DevTensor*>(d_workspace), (int)v.size(), (uint32_t)groups, d_status);
  }
  if (cudaGetLastError() != cudaSuccess) return ECF8_ERR_CUDA;
  g_launches.fetch_add(1);
  return ECF8_OK;
}

uint64_t ecf8_launch_count(void) { return g_launches.load(); }

}  // extern "C"

// ---------------------------------------------------------------- no-allocation batched decode
//
// The descriptor table of ecf8_decode_batched_noalloc.  It is device memory
// the library owns (one copy per GPU that loads the library), so callers that
// cannot allocate need not pass a workspace.  In host code the name
// g_noalloc_table stands for the host-side shadow of the symbol, not a device
// address: the device address is looked up with cudaGetSymbolAddress, once
// per device, and that pointer is what the kernel receives.  Nothing in the
// table needs to start at zero: every call writes the entries it uses.
namespace ecf8 {
namespace {

static __device__ __align__(256) DevTensor g_noalloc_table[ECF8_NOALLOC_MAX_TENSORS];

// Device address of g_noalloc_table on the current device (resolved on the
// first call there, with that device current).
int noalloc_table_address(DevTensor** out) {
  static std::atomic<DevTensor*> per_dev[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ECF8_ERR_CUDA;
  DevTensor* p = per_dev[dev].load();
  if (!p) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_noalloc_table) != cudaSuccess || !addr) return ECF8_ERR_CUDA;
    p = static_cast<DevTensor*>(addr);
    per_dev[dev].store(p);
  }
  *out = p;
  return ECF8_OK;
}

}  // namespace
}  // namespace ecf8

extern "C" int ecf8_decode_batched_noalloc(const ecf8_tensor* tensors, int count, int32_t* d_status,
                                           cudaStream_t s) {
  if (count < 0 || (count > 0 && !tensors)) return ECF8_ERR_ARG;
  if (count == 0) return ECF8_OK;
  if (count > ECF8_NOALLOC_MAX_TENSORS) return ECF8_ERR_TOO_MANY;
  // host staging of the descriptors: a fixed array, reused under a lock; the
  // pageable host->device copy has read it by the time cudaMemcpyAsync returns
  static DevTensor host_table[ECF8_NOALLOC_MAX_TENSORS];
  static std::mutex host_lock;
  std::lock_guard<std::mutex> guard(host_lock);
  int used = 0;
  uint64_t groups = 0;
  for (int i = 0; i < count; ++i) {
    const ecf8_info* info = tensors[i].info;
    int rc = check_info(info);
    if (rc) return rc;
    if (info->chunk_bytes != (uint32_t)kC || info->group_chunks != (uint32_t)kT) return ECF8_ERR_UNSUPPORTED;
    if (info->n == 0) continue;
    if (!tensors[i].d_blob || !tensors[i].d_out) return ECF8_ERR_ARG;
    if (!aligned16(tensors[i].d_blob) || !aligned16(tensors[i].d_out)) return ECF8_ERR_ALIGN;
    DevTensor t = make_dev(info, tensors[i].d_blob, tensors[i].d_out);
    t.group_base = (uint32_t)groups;
    groups += info->n_groups;
    if (groups > 0xFFFFFFFFull) return ECF8_ERR_UNSUPPORTED;
    host_table[used++] = t;
  }
  if (used == 0) return ECF8_OK;
  DevTensor* table = nullptr;
  int rc = noalloc_table_address(&table);
  if (rc) return rc;
  uint32_t ctas = 0;
  if ((rc = grid_for_device<kC, kT>(&ctas))) return rc;
  if (cudaMemcpyAsync(table, host_table, sizeof(DevTensor) * (size_t)used, cudaMemcpyHostToDevice, s) !=
      cudaSuccess)
    return ECF8_ERR_CUDA;
  decode_table_kernel<kC, kT><<<grid_size(ctas, groups), kT, Shape<kC, kT>::kSmemBytes, s>>>(table, used,
                                                                                              (uint32_t)groups,
                                                                                              d_status);
  if (cudaGetLastError() != cudaSuccess) return ECF8_ERR_CUDA;
  g_launches.fetch_add(1);
  return ECF8_OK;
}
