// ECF8 GPU decoder for sm_100a.
//
// Reconstructs FP8 E4M3 bytes from a Huffman-coded exponent stream and a
// sign/mantissa nibble array (ECF8 walkthrough "ECF8 浮点数压缩技术" §3.2.1, the
// decode_kernel pipeline; arXiv 2510.02676 abstract).  The pages' kernel is
// prior art written for H100/RTX40 parts; this one keeps its idea -- every
// thread owns a fixed slice of the bit stream, starts at a stored gap, counts
// its codes, and a prefix sum of the counts places its output -- and is
// otherwise laid out for B200:
//
//  * a group is 32 chunks of 32 stream bytes and belongs to ONE warp: the
//    warp's lanes decode its chunks, a warp-shuffle scan of their code counts
//    added to the group's stored offset places every exponent, and the warp
//    writes the group's output.  Warps never wait for each other; the only
//    CTA-wide barriers sit where a CTA's run of groups enters a new tensor.
//  * decoding is a finite-state machine over bytes: a 4096-entry table in
//    shared memory, indexed by (node of the code tree, next stream byte),
//    gives every exponent whose code ends in that byte and the node after
//    it.  Entries are 64-bit when the code has a 1-bit length (up to 8 codes
//    end in a byte) and 32-bit otherwise (at most 4), which halves the banks
//    a warp's random lookups touch; the narrow walk also packs two bytes'
//    exponents per step.  Each lane first shifts its slice so that it starts
//    at its first code (the gap), and zeroes the bits after its last code, so
//    all lanes run the same fully unrolled 34-byte loop.  Zeros after a code
//    boundary decode as repeats of the all-zero code, whose number is known
//    and subtracted.
//  * exponents are parked 4 bits each in lane-private shared memory, then
//    funnel-shifted into a 32-weight-aligned stage; 16 bytes of stage plus a
//    16-byte nibble load become 32 output bytes (per 8 weights two shifts,
//    a rotate and two 3-input bit-selects: the blob's code order and nibble
//    words put every field where its output byte wants it), and consecutive
//    lanes store consecutive 32-byte vectors.
//  * CTAs are persistent, one per SM.  A launch puts the wide-table tensors on
//    CTAs [0, split) and the rest on the others; within each part every CTA
//    takes a contiguous run of groups of equal estimated cost.  Every warp
//    fetches its next group's stream slice, gaps and offsets while it decodes
//    the current one, and issues the current group's nibble loads before its
//    walk.  Launches allow programmatic dependent launch, so a decode builds
//    its first table while the previous kernel on the stream drains.
//
// The path is HBM-bound integer work: no tensor cores.  Corrupt input is
// reported through a status word; no access leaves its buffer and no loop
// runs without a bound.
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "ecf8.h"
#include "ecf8_format.h"

namespace ecf8 {
namespace {

// Layout the kernels implement: 32-byte chunks, 32 chunks (one warp) per group.
constexpr int kC = 32, kT = 32;
constexpr int kWords = kC / 4;                 // stream words per chunk
constexpr int kSpanBits = 8 * kC;              // 256
constexpr int kBytes = (kSpanBits + 15 + 7) / 8 + 0;  // 34: a lane may own up to 256 + 15 bits
static_assert(kBytes % 2 == 0, "the narrow walk takes bytes in pairs");
constexpr int kPadBits = 8 * kBytes;           // 272 bits walked by every lane
constexpr int kPrivWords = kBytes + 1;         // parked exponent words per lane (<= 272 codes)
constexpr int kMaxCodes = kSpanBits * kT;      // codes one group can hold: 8192
constexpr int kStageWords = kMaxCodes / 8 + 8; // + alignment slack
constexpr int kStagePhys = kStageWords + 2 * (kStageWords / 32 + 1) + 2;  // 2 pad words per 32

// Tuning knobs (compile-time; the defaults are the measured best on B200).
#ifndef ECF8_WARPS
#define ECF8_WARPS 16
#endif
#ifndef ECF8_NIB_PREFETCH
#define ECF8_NIB_PREFETCH 4
#endif
#ifndef ECF8_PREFETCH_NEXT
#define ECF8_PREFETCH_NEXT 1
#endif

constexpr int kWarps = ECF8_WARPS;             // warps per CTA
constexpr int kThreads = 32 * kWarps;
constexpr int kND = ECF8_NIB_PREFETCH;         // 32-weight nibble blocks a lane prefetches in registers
constexpr int kNDA = kND > 0 ? kND : 1;        // their array size
constexpr bool kPrefetchNext = ECF8_PREFETCH_NEXT != 0;  // fetch the next group's inputs during this one
constexpr int kStates = 16;                    // tree nodes (<= 15 for 16 values) + the error state
constexpr int kError = kStates - 1;

// Shared memory of one CTA.  Every member read as a 16-byte vector starts on
// a 16-byte boundary (checked below).
struct alignas(16) Tree {
  uint32_t first[17], count[17], base[17];  // canonical code per length
  uint32_t nint[17], ibase[17];             // internal nodes per depth, their first state id
  uint32_t nstates, max_len, ok, lmin;
  uint8_t sorted[16];
  uint16_t bit_step[kStates * 2];            // (state, bit) -> next state | symbol << 4 | emitted << 8
  uint32_t nib_step[kStates * 16];           // (state, 4 bits) -> symbols | count << 16 | next << 20
  uint16_t zero_codes[kPadBits + 1];         // codes in k zero bits after a code boundary
};
struct alignas(16) WarpArea {
  uint32_t priv[kPrivWords * 32];  // word k of lane l at k*32 + l
  uint32_t stage[kStagePhys];      // word w at sidx(w); read as uint2 per 16-weight unit
};
struct alignas(16) Smem {
  // the byte table, indexed by node << 8 | byte.  Wide entries (any code):
  // x = exponents (4 bits each, first lowest), y = next node | 4*count << 8.
  // Narrow entries (shortest code >= 2 bits, so <= 4 codes end in a byte;
  // the first 16 KB): exponents in bits 0-15, next node in bits 16-23,
  // 4*count in bits 24-31.
  uint2 fsm[kStates * 256];
  Tree tree;
  WarpArea warp[kWarps];
};
static_assert(offsetof(WarpArea, stage) % 16 == 0, "stage must be 16-byte aligned");
static_assert(sizeof(WarpArea) % 16 == 0, "warp areas must stay 16-byte aligned");
static_assert(offsetof(Smem, warp) % 16 == 0, "warp areas must be 16-byte aligned");
static_assert(offsetof(Smem, fsm) % 16 == 0, "table must be aligned");
static_assert(sizeof(Smem) <= 227 * 1024, "shared memory budget");

// Checked builds (-DECF8_CHECKED, libecf8_checked.so) test each index a
// store or a table read uses against its buffer; a failing one skips the
// access and sets ECF8_STATUS_BOUNDS.  Release builds compile the tests away.
#ifdef ECF8_CHECKED
__device__ __forceinline__ bool in_bounds(bool ok, int32_t* status) {
  if (!ok && status) atomicOr(status, ECF8_STATUS_BOUNDS);
  return ok;
}
#else
__device__ __forceinline__ bool in_bounds(bool, int32_t*) { return true; }
#endif

// ---------------------------------------------------------------- decode tables

// Canonical code and internal-node numbering, by one warp.  State 0 is the
// root; the internal nodes at depth l are the values first[l] + count[l] + k,
// k < nint[l], numbered from ibase[l].  Lane s < 16 holds symbol s's length;
// lane l in 1..16 counts the codes of length l; a symbol's place in the
// canonical order is its length's base plus its rank among the symbols of
// that length.  Only the two 16-step recurrences (first codes, internal
// nodes per depth) run on lane 0.
__device__ void build_tree(const uint8_t* len, Tree* t) {
  const uint32_t lane = threadIdx.x & 31;
  const uint32_t L = lane < 16 ? len[lane] : 0u;
  uint32_t cnt = 0;
#pragma unroll
  for (uint32_t l = 1; l <= 16; ++l) {
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, L == l);
    if (lane == l) cnt = __popc(m);
  }
  uint32_t incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= (uint32_t)o) incl += v;
  }
  const uint32_t base = incl - cnt;  // lane l: codes shorter than l
  const uint32_t my_base = __shfl_sync(0xFFFFFFFFu, base, L & 31u);
  const uint32_t same = __match_any_sync(0xFFFFFFFFu, L);
  const uint32_t rank = __popc(same & ((1u << lane) - 1u));
  if (lane < 16 && L) t->sorted[my_base + rank] = (uint8_t)lane;
  if (lane <= 16) {
    t->count[lane] = cnt;
    t->base[lane] = base;
  }
  const uint32_t max_len = __reduce_max_sync(0xFFFFFFFFu, L);
  const uint32_t present = __popc(__ballot_sync(0xFFFFFFFFu, L != 0));
  const uint32_t kraft = __reduce_add_sync(0xFFFFFFFFu, (L && L <= 16) ? 1u << (16 - L) : 0u);
  const uint32_t lmin = __reduce_min_sync(0xFFFFFFFFu, L ? L : 99u);
  __syncwarp();
  if (lane == 0) {
    uint32_t code = 0;
    t->first[0] = 0;
#pragma unroll
    for (int l = 1; l <= 16; ++l) {
      code = (code + t->count[l - 1]) << 1;
      t->first[l] = code;
    }
    int ok = present == 1 || kraft == (1u << 16);
    t->nint[0] = 1;
    t->ibase[0] = 0;
    uint32_t states = 1, prev = 1;
#pragma unroll
    for (uint32_t l = 1; l <= 16; ++l) {
      int n = l < max_len ? 2 * (int)prev - (int)t->count[l] : 0;
      if (n < 0) {
        ok = 0;
        n = 0;
      }
      t->nint[l] = (uint32_t)n;
      t->ibase[l] = states;
      states += (uint32_t)n;
      prev = (uint32_t)n;
    }
    if (states > kStates - 1) ok = 0;
    t->nstates = states;
    t->max_len = max_len;
    t->ok = ok;
    t->lmin = lmin <= 16 ? lmin : 1;  // the all-zero path from the root meets a code after lmin zeros
  }
}

// One bit from tree node `state`: the next node, and the value whose code
// it completes (if any); the error state absorbs everything.
__device__ uint32_t bit_entry(const Tree* t, uint32_t state, uint32_t bit) {
  if (!t->ok || state >= t->nstates) return kError;
  uint32_t l = 0, v = 0;
  for (uint32_t d = 1; d < t->max_len; ++d)
    if (state >= t->ibase[d] && state < t->ibase[d] + t->nint[d]) {
      l = d;
      v = t->first[d] + t->count[d] + (state - t->ibase[d]);
    }
  v = 2 * v + bit;
  ++l;
  const uint32_t r = v - t->first[l];
  if (r < t->count[l]) return 0u | ((uint32_t)t->sorted[t->base[l] + r] << 4) | (1u << 8);  // back to the root
  if (l >= t->max_len) return kError;
  return t->ibase[l] + (v - t->first[l] - t->count[l]);
}

// Table widths: a tensor whose shortest code is 1 bit can end 8 codes in one
// byte and needs the wide table; any other fits the narrow one, whose
// lookups touch half the shared-memory banks of wide ones.
constexpr int kWide = 64, kNarrow = 32;

// K0: the tensor's tables into shared memory (all threads of the CTA):
// bit steps -> 4-bit steps -> the byte table, each built from the last.
template <int kW>
__device__ void load_tables(const DevTensor* dt, Smem* sm) {
  Tree* t = &sm->tree;
  const int tid = threadIdx.x;
  __syncthreads();  // every warp is done with the previous tensor's tables
  if (tid < 32) build_tree(dt->len, t);
  __syncthreads();
  if (tid < kStates * 2) t->bit_step[tid] = (uint16_t)bit_entry(t, tid >> 1, tid & 1);
  for (int z = tid; z <= kPadBits; z += kThreads) t->zero_codes[z] = (uint16_t)(z / t->lmin);
  __syncthreads();
  if (tid < kStates * 16) {
    uint32_t st = tid >> 4, syms = 0, n = 0;
    for (int i = 3; i >= 0; --i) {
      const uint32_t e = t->bit_step[2 * st + ((tid >> i) & 1)];
      if (e & 0x100) syms |= ((e >> 4) & 15u) << (4 * n++);
      st = e & 15u;
    }
    t->nib_step[tid] = syms | (n << 16) | (st << 20);
  }
  __syncthreads();
  for (int e = tid; e < kStates * 256; e += kThreads) {
    const uint32_t a = t->nib_step[((e >> 8) << 4) | ((e >> 4) & 15)];
    const uint32_t na = (a >> 16) & 15u, sa = a >> 20;
    const uint32_t b = t->nib_step[(sa << 4) | (e & 15)];
    const uint32_t nb = (b >> 16) & 15u, sb = b >> 20;
    const uint32_t syms = (a & 0xFFFFu) | ((b & 0xFFFFu) << (4 * na));
    const uint32_t n4 = 4 * (na + nb);
    if (kW == kWide)
      sm->fsm[e] = sb == (uint32_t)kError ? make_uint2(0, kError) : make_uint2(syms, sb | (n4 << 8));
    else
      reinterpret_cast<uint32_t*>(sm->fsm)[e] = sb == (uint32_t)kError ? (uint32_t)kError << 16
                                                                       : (syms & 0xFFFFu) | (sb << 16) | (n4 << 24);
  }
  __syncthreads();
}

// With the wide table, stage word w lives at w + 2*(w/32): when nearly every
// code is 1 bit long, lanes' runs start 32 words apart and would otherwise
// all store to one bank.  Word pairs (2u, 2u+1) stay adjacent and 8-byte
// aligned.  With the narrow table (codes >= 2 bits) the plain layout spreads
// the lanes' stores better.
template <int kW>
__device__ __forceinline__ uint32_t sidx(uint32_t w) { return kW == kWide ? w + ((w >> 5) << 1) : w; }
template <int kW>  // uint2 index of unit u
__device__ __forceinline__ uint32_t sunit(uint32_t u) { return kW == kWide ? u + (u >> 4) : u; }

// Index of a narrow-table entry: byte k of stream word w, then the node held
// in byte 2 of entry e; the upper bytes replicate that byte's sign bit, which
// is zero since nodes are < 16 (prmt's sign-replicate selector nibbles).
__device__ __forceinline__ uint32_t nidx(uint32_t w, uint32_t e, uint32_t k) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(w), "r"(e), "r"(0xEE60u | k));
  return r;
}

// ---------------------------------------------------------------- assembly

// Bits 3-6 of every byte from a, the others from b: one 3-input logic op.
__device__ __forceinline__ uint32_t merge_exp(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, 0x78787878, 0xE4;" : "=r"(r) : "r"(a), "r"(b));  // (a & c) | (b & ~c)
  return r;
}

// 8 weights of a whole block: E = their exponents in stream order, so byte k
// of E holds weight k's exponent in its low nibble and weight 4+k's in its
// high nibble; N = their nibble word (byte k: weight k's sign in bit 7 and
// mantissa in bits 0-2, weight 4+k's mantissa in bits 4-6, weight
// 4+((k+3)%4)'s sign in bit 3).  Weights 0-3: E << 3 puts each low nibble
// at bits 3-6, N has the rest in place; weights 4-7: E >> 1 and N rotated
// right by 4.
__device__ __forceinline__ void assemble8(uint32_t E, uint32_t N, uint32_t& lo, uint32_t& hi) {
  lo = merge_exp(E << 3, N);
  hi = merge_exp(E >> 1, __funnelshift_r(N, N, 4));
}

// 32 weights from their exponents (4 words, 8 per word) and nibbles (16
// bytes), stored with one 32-byte store when the destination allows it.
__device__ __forceinline__ void put32(uint8_t* dst, bool a32, uint4 ex, uint4 nb) {
  uint32_t o[8];
  assemble8(ex.x, nb.x, o[0], o[1]);
  assemble8(ex.y, nb.y, o[2], o[3]);
  assemble8(ex.z, nb.z, o[4], o[5]);
  assemble8(ex.w, nb.w, o[6], o[7]);
  if (a32) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(o[0]), "r"(o[1]),
                 "r"(o[2]), "r"(o[3]), "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7])
                 : "memory");
  } else {
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(o[0], o[1], o[2], o[3]);
    reinterpret_cast<uint4*>(dst)[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// Exponents of the 32-weight block d (units 2d, 2d+1) from the stage.
template <int kW>
__device__ __forceinline__ uint4 stage32(const uint32_t* stage, uint32_t d) {
  if (kW == kNarrow) return reinterpret_cast<const uint4*>(stage)[d];
  const uint2* st = reinterpret_cast<const uint2*>(stage);
  const uint2 a = st[sunit<kW>(2 * d)], b = st[sunit<kW>(2 * d + 1)];
  return make_uint4(a.x, a.y, b.x, b.y);
}

// The walk's packer step: when the accumulator has filled a word (sh >= 32),
// park it as the lane's next private word and keep the carry.
__device__ __forceinline__ void park(uint32_t& sh, uint32_t* priv, uint32_t& words, uint32_t& acc, uint32_t carry,
                                     int32_t* status) {
  const bool full = sh >= 32;
  if (full && in_bounds(words < (uint32_t)kPrivWords, status)) priv[32 * words] = acc;
  words += full ? 1u : 0u;
  acc = full ? carry : acc;
  sh -= full ? 32u : 0u;
}

// ---------------------------------------------------------------- one group per warp

// What a lane fetches ahead for a group: its slice + the next word (a code
// may run past the slice end), the raw gap word(s), the group's offsets.
// Kept raw so the loads stay in flight until used.
struct GroupIn {
  uint32_t w[kWords + 1];
  uint32_t gapw, gapn;
  uint64_t off0, off1;
};

__device__ __forceinline__ void fetch_group(const DevTensor* dt, uint32_t local, GroupIn& in) {
  const uint32_t lane = threadIdx.x & 31;
  const uint64_t chunk = (uint64_t)local * kT + lane;
  // inside a group the stream is stored word-major (word m of chunk c at
  // m * kT + c): the warp's load of word m is 128 contiguous bytes.  A lane's
  // next word is word 0 of the next chunk, stored right after its own word 0;
  // lane 31's is word 0 of the next group's first chunk (or the stream's zero
  // tail after the last group)
  const uint32_t* gs = dt->stream + (uint64_t)local * (kT * kWords) + lane;
#pragma unroll
  for (int m = 0; m < kWords; ++m) in.w[m] = __ldg(gs + m * kT);
  in.w[kWords] = __ldg(gs + (lane + 1 < (uint32_t)kT ? 1u : (uint32_t)(kT * kWords - lane)));
  in.gapw = __ldg(dt->gaps + (chunk >> 3));
  // the first gap of the next group (lane 31's right neighbour), if it exists
  in.gapn = (lane == 31 && local + 1 < dt->n_groups) ? __ldg(dt->gaps + ((chunk + 1) >> 3)) : 0u;
  in.off0 = __ldg(dt->groups + local);
  in.off1 = __ldg(dt->groups + local + 1);
}

template <int kW>
__device__ __forceinline__ void process_group(const DevTensor* dt, uint32_t local, const GroupIn& in, Smem* sm,
                                              WarpArea* wa, int32_t* status) {
  const uint32_t lane = threadIdx.x & 31;
  const uint64_t n = dt->n;
  const uint64_t off0 = in.off0, off1 = in.off1;
  const bool offsets_ok = off0 <= off1 && off1 <= n && off1 - off0 <= (uint64_t)kMaxCodes;

  // this group's nibbles: issued now, consumed after the walk
  // (16-weight units: unit u = weights base + 16u.., 8 bytes of nibbles,
  // base = off0 rounded down to 32); also the nibble words of the group's
  // first and last unit when the group owns them only in part
  const uint32_t units = offsets_ok ? (uint32_t)(((off0 & 31) + (off1 - off0) + 15) >> 4) : 0;
  const uint32_t blocks = (units + 1) >> 1;  // 32-weight blocks: 16 nibble bytes each
  const uint4* nib = reinterpret_cast<const uint4*>(dt->nibbles) + (off0 >> 5);
  uint4 nv[kNDA];
#pragma unroll
  for (int j = 0; j < kND; ++j)
    if (lane + 32 * j < blocks && in_bounds((off0 >> 5) + lane + 32 * j < (n + 31) / 32, status))
      nv[j] = __ldg(nib + lane + 32 * j);
  const uint32_t* nib32 = reinterpret_cast<const uint32_t*>(nib);
  const uint32_t u0 = (uint32_t)(off0 & 31) >> 4;
  const uint32_t first_full = u0 + ((off0 & 15) ? 1u : 0u);
  const uint32_t end_full = (units && (off1 & 15)) ? units - 1 : units;
  const bool hr = units && first_full != u0;  // units == 0 when the offsets are not to be trusted
  const bool tr = end_full < units && !(hr && end_full == u0);
  // the ragged units' nibble words: lanes 0-15 the head's, lanes 16-31 the tail's
  const bool rg = lane < 16 ? hr : tr;
  const uint32_t ru = lane < 16 ? u0 : end_full;
  const uint32_t rw = rg ? __ldg(nib32 + 2 * ru + ((lane & 15) >> 3)) : 0u;

  // K1: the lane's bits run from its first code (gap) to the next lane's
  // first code, or to the stream end: E bits once shifted to start at 0
  const uint32_t gap = (in.gapw >> ((lane & 7) * 4)) & 15u;
  uint32_t gap_next = __shfl_down_sync(0xFFFFFFFFu, gap, 1);
  if (lane == 31) gap_next = in.gapn & 15u;
  const uint64_t bit0 = ((uint64_t)local * kT + lane) * kSpanBits;
  const uint64_t code_bits = dt->code_bits;
  const uint64_t left = bit0 < code_bits ? code_bits - bit0 : 0;
  const uint32_t stop = left < (uint64_t)(kSpanBits + gap_next) ? (uint32_t)left : kSpanBits + gap_next;
  const uint32_t E = stop > gap ? stop - gap : 0;
  uint32_t sw[kWords + 1];
#pragma unroll
  for (int i = 0; i < kWords; ++i) sw[i] = __funnelshift_l(in.w[i + 1], in.w[i], gap);
  sw[kWords] = in.w[kWords] << gap;
  // zero every bit at or after E (bits 32i.. of sw[i]); a lane that is not at
  // the stream end keeps E >= 241, so only its last two words need it
  const bool any_short = __any_sync(0xFFFFFFFFu, E < 32 * (kWords - 1));
#pragma unroll
  for (int i = 0; i <= kWords; ++i) {
    if (i >= kWords - 1 || any_short) {
      const int keep = min(max((int)E - 32 * i, 0), 32);
      sw[i] &= (uint32_t)(0xFFFFFFFF00000000ull >> keep);
    }
  }

  // K2: the byte machine.  Every lane walks 272 bits; codes completed in the
  // zero bits after E are repeats of the all-zero code and are subtracted.
  uint32_t* priv = wa->priv + lane;
  uint32_t y = 0;  // previous entry's node | count word (root, none)
  uint32_t acc = 0, sh = 0, words = 0;
  if (kW == kWide) {
#pragma unroll
    for (int j = 0; j < kBytes; ++j) {
      const uint32_t idx = __byte_perm(sw[j >> 2], y, 0x7740u | (3u - (j & 3)));  // byte | node << 8
      const uint2 e = in_bounds(idx < (uint32_t)(kStates * 256), status) ? sm->fsm[idx] : make_uint2(0, kError);
      y = e.y;
      acc |= e.x << sh;
      const uint32_t carry = __funnelshift_l(e.x, 0u, sh);
      sh += e.y >> 8;
      park(sh, priv, words, acc, carry, status);
    }
  } else {
    // two bytes per packing step: each ends at most 4 codes (16 bits), so a
    // pair's exponents fit one word
    const uint32_t* tab = reinterpret_cast<const uint32_t*>(sm->fsm);
#pragma unroll
    for (int j = 0; j < kBytes; j += 2) {
      const uint32_t i1 = nidx(sw[j >> 2], y, 3u - (j & 3));
      const uint32_t e1 = in_bounds(i1 < (uint32_t)(kStates * 256), status) ? tab[i1] : (uint32_t)kError << 16;
      const uint32_t i2 = nidx(sw[(j + 1) >> 2], e1, 3u - ((j + 1) & 3));
      const uint32_t e2 = in_bounds(i2 < (uint32_t)(kStates * 256), status) ? tab[i2] : (uint32_t)kError << 16;
      y = e2;
      const uint32_t n1 = e1 >> 24;
      const uint32_t p = (e1 & 0xFFFFu) | ((e2 & 0xFFFFu) << n1);
      acc |= p << sh;
      const uint32_t carry = __funnelshift_l(p, 0u, sh);
      sh += n1 + (e2 >> 24);
      park(sh, priv, words, acc, carry, status);
    }
  }
  if (sh && in_bounds(words < (uint32_t)kPrivWords, status)) priv[32 * words] = acc;
  const uint32_t emitted = 8 * words + sh / 4;
  const uint32_t extra = sm->tree.zero_codes[kPadBits - E];
  const uint32_t node = kW == kWide ? y & 0xFFu : (y >> 16) & 0xFFu;
  const bool bad = node == (uint32_t)kError || emitted < extra;
  const uint32_t cnt = bad ? 0 : emitted - extra;

  // the rest of a group of many short codes, once the walk's registers are free
  uint4 nv2[kNDA];
  if (kND > 0 && kW == kWide && blocks > 32u * kND) {
#pragma unroll
    for (int j = 0; j < kND; ++j)
      if (lane + 32 * (kND + j) < blocks && in_bounds((off0 >> 5) + lane + 32 * (kND + j) < (n + 31) / 32, status))
        nv2[j] = __ldg(nib + lane + 32 * (kND + j));
  }

  // K3: place -- warp-shuffle scan of the counts
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
    return;  // uniform across the warp
  }

  // K4a: funnel-shift this lane's exponents to stage nibble position
  // (off0 mod 32) + start, so that stage words 4b..4b+3 cover output block b.
  // Words shared with a neighbour lane are zeroed, then OR-ed atomically.
  uint32_t* stage = wa->stage;
  const uint32_t q = (uint32_t)(off0 & 31) + start;
  const uint32_t d0 = q >> 3, dl = cnt ? (q + cnt - 1) >> 3 : 0;
  if (cnt) {
    if (in_bounds(sidx<kW>(dl) < (uint32_t)kStagePhys, status)) {
      stage[sidx<kW>(d0)] = 0;
      stage[sidx<kW>(dl)] = 0;
    }
  }
  __syncwarp();
  if (cnt) {
    const uint32_t r = (q & 7) * 4;
    const uint32_t used = (cnt + 7) / 8;
    // the last parked word may hold padding codes after the lane's own ones
    if (cnt & 7) priv[32 * (used - 1)] &= (1u << (4 * (cnt & 7))) - 1;
    const uint32_t nwd = dl - d0 + 1;  // destination words: used or used + 1
    uint32_t prev = priv[0];
    if (in_bounds(sidx<kW>(d0) < (uint32_t)kStagePhys, status)) atomicOr(&stage[sidx<kW>(d0)], prev << r);
    uint32_t j = 1;
    if (kW == kNarrow) {
      // codes of 2 bits or more: at most 135 per lane, so at most 16
      // interior words; a fully unrolled, predicated loop
#pragma unroll
      for (uint32_t k = 1; k <= 16; ++k) {
        const uint32_t cur = priv[32 * k];
        if (k + 1 < nwd && in_bounds(sidx<kW>(d0 + k) < (uint32_t)kStagePhys, status))
          stage[sidx<kW>(d0 + k)] = __funnelshift_l(prev, cur, r);
        prev = cur;
      }
      j = nwd > 1 ? nwd - 1 : 1;
      prev = priv[32 * (j - 1)];
    } else {
#pragma unroll 4
      for (; j + 1 < nwd; ++j) {  // interior words belong to this lane alone
        const uint32_t cur = priv[32 * j];
        if (in_bounds(sidx<kW>(d0 + j) < (uint32_t)kStagePhys, status))
          stage[sidx<kW>(d0 + j)] = __funnelshift_l(prev, cur, r);
        prev = cur;
      }
    }
    if (nwd > 1) {
      const uint32_t cur = j < used ? priv[32 * j] : 0;
      if (in_bounds(sidx<kW>(d0 + j) < (uint32_t)kStagePhys, status))
        atomicOr(&stage[sidx<kW>(d0 + j)], __funnelshift_l(prev, cur, r));
    }
  }
  __syncwarp();

  // K4b + K5: whole 32-weight blocks by their lane -- consecutive lanes store
  // consecutive 32 bytes, 1 KB contiguous per instruction; a whole unit
  // whose block is not whole (at most one at each end) by lane 0 or 1; the
  // ragged first and last unit one byte per lane
  const uint64_t base = off0 & ~31ull;
  uint8_t* out = dt->out;
  const bool a32 = ((reinterpret_cast<uintptr_t>(out) & 31) == 0);
#pragma unroll
  for (int j = 0; j < kND; ++j) {
    const uint32_t d = lane + 32 * j;
    if (2 * d + 2 <= end_full && (j > 0 || 2 * d >= first_full))  // first_full <= 2
      if (in_bounds(base + 32ull * d + 32 <= n, status)) put32(out + base + 32ull * d, a32, stage32<kW>(stage, d), nv[j]);
  }
  if (kND > 0 && kW == kWide && end_full > 64u * kND) {
#pragma unroll
    for (int j = 0; j < kND; ++j) {
      const uint32_t d = lane + 32 * (kND + j);
      if (2 * d + 2 <= end_full && in_bounds(base + 32ull * d + 32 <= n, status))
        put32(out + base + 32ull * d, a32, stage32<kW>(stage, d), nv2[j]);
    }
  }
  for (uint32_t d = lane + 32 * (kW == kWide ? 2 * kND : kND); 2 * d + 2 <= end_full; d += 32)
    if ((kND > 0 || 2 * d >= first_full) && in_bounds(base + 32ull * d + 32 <= n, status))
      put32(out + base + 32ull * d, a32, stage32<kW>(stage, d), __ldg(nib + d));
  {
    // a whole unit whose block partner is not whole: unit first_full when it
    // is odd (lane 0), unit end_full - 1 when end_full is odd (lane 1)
    uint32_t su = ~0u;
    if (lane == 0 && (first_full & 1) && first_full < end_full) su = first_full;
    if (lane == 1 && (end_full & 1) && end_full - 1 >= first_full) su = end_full - 1;
    if (su != ~0u) {
      const uint2 ex = reinterpret_cast<const uint2*>(stage)[sunit<kW>(su)];
      const uint2 nb = reinterpret_cast<const uint2*>(nib)[su];
      uint32_t o[4];
      assemble8(ex.x, nb.x, o[0], o[1]);
      assemble8(ex.y, nb.y, o[2], o[3]);
      if (in_bounds(base + 16ull * su + 16 <= n, status))
        *reinterpret_cast<uint4*>(out + base + 16ull * su) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  if (hr || tr) {
    // weight p's code sits at stream position s: the group writes the weights
    // whose codes it holds, the neighbouring group the others
    const uint64_t p = base + 16ull * ru + (lane & 15);
    const uint64_t s = code_position(p, n);
    if (rg && s >= off0 && s < off1) {
      const uint32_t i = (uint32_t)(s - base);
      const uint32_t e = (stage[sidx<kW>(i >> 3)] >> (4 * (i & 7))) & 15u;
      const uint32_t k = lane & 7;
      const uint32_t half = k < 4 ? rw : __funnelshift_r(rw, rw, 4);
      const uint32_t v = (half >> (8 * (k & 3))) & 0x87u;
      if (in_bounds(p < n, status)) out[p] = (uint8_t)(v | (e << 3));
    }
  }
  __syncwarp();  // the stage and private words are reused by this warp's next group
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

// A CTA that enters a new tensor part way through its run rebuilds its table
// and first waits for all its warps to finish the previous tensor: each
// tensor's cost range starts with this much (about 18 groups' worth), so such
// CTAs take fewer groups.
constexpr uint64_t kTensorSetupCost = 100000;

// The group that starts at estimated cost c of the launch: in the tensor whose
// cost range holds c, the first group whose cost range starts at or after c.
// Non-decreasing in c, 0 at c = 0 and the launch's group count at its total
// cost, so consecutive cost cuts give disjoint group runs that cover all.
__device__ __forceinline__ uint32_t group_at_cost(const DevTensor* ts, int count, uint64_t c) {
  int lo = 0, hi = count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ts[mid].cost_base <= c) lo = mid;
    else hi = mid - 1;
  }
  const uint64_t w = ts[lo].group_cost, rel = c - ts[lo].cost_base;
  uint64_t k = rel > kTensorSetupCost ? (rel - kTensorSetupCost + w - 1) / w : 0;
  if (k > ts[lo].n_groups) k = ts[lo].n_groups;
  return ts[lo].group_base + (uint32_t)k;
}

// Persistent CTA over a contiguous run of groups (across tensors, in table
// order) holding an equal share of the launch's estimated cost: a group of a
// tensor with short codes holds more weights and takes longer.  Within each
// tensor's part of the run, warp w takes groups w, w+W, ... and fetches its
// next group while decoding the current one.
// Programmatic dependent launch: the next kernel on the stream may start its
// CTAs (on SMs this launch has left) before this grid ends; a decode builds
// its first table from the codebook in its parameters before it waits for
// the previous grid, whose writes it may read (blobs) or overwrite (outputs).
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void wait_prerequisites() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <int kW>
__device__ __forceinline__ void decode_run(const DevTensor* table, int count, uint32_t total, uint64_t total_cost,
                                           uint32_t cta, uint32_t ctas, int32_t* status) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Smem* sm = reinterpret_cast<Smem*>(smem_raw);
  const uint32_t gb = group_at_cost(table, count, (uint64_t)cta * total_cost / ctas);
  const uint32_t ge =
      cta + 1 == ctas ? total : group_at_cost(table, count, (uint64_t)(cta + 1) * total_cost / ctas);
  if (gb >= ge) return;
  const uint32_t warp = threadIdx.x >> 5;
  WarpArea* wa = &sm->warp[warp];
  int ti = find_tensor(table, count, gb);
  uint32_t g0 = gb;
  while (g0 < ge) {
    const DevTensor* dt = table + ti;
    const uint32_t tb = dt->group_base, te = tb + dt->n_groups;
    const uint32_t g1 = te < ge ? te : ge;  // this tensor's part of the run: [g0, g1)
    load_tables<kW>(dt, sm);
    if (g0 == gb) wait_prerequisites();  // once, after the first table
    uint32_t g = g0 + warp;
    if (g < g1) {
      GroupIn in;
      if (kPrefetchNext) fetch_group(dt, g - tb, in);
      for (; g < g1; g += kWarps) {
        GroupIn nx;
        const bool more = g + kWarps < g1;
        if (!kPrefetchNext) fetch_group(dt, g - tb, in);
        else if (more) fetch_group(dt, g + kWarps - tb, nx);
        process_group<kW>(dt, g - tb, in, sm, wa, status);
        if (kPrefetchNext && more) in = nx;
      }
    }
    g0 = g1;
    ++ti;
  }
}

// The two parts of a launch: the tensors that need the wide table come
// first in the descriptor table and are decoded by CTAs [0, split); the
// others, from descriptor `first` on, by CTAs [split, grid).  Each part
// spreads its own estimated cost evenly over its CTAs.  The branch on the
// part is taken once per CTA, so each part's code keeps its own registers.
struct PartArgs {
  int first, count;
  uint32_t groups;
  uint64_t cost;
};
struct SplitArgs {
  uint32_t split;
  PartArgs part[2];
};

__device__ __forceinline__ void decode_split(const DevTensor* t, const SplitArgs& a, int32_t* status) {
  if (blockIdx.x < a.split) {
    const PartArgs& p = a.part[0];
    decode_run<kWide>(t + p.first, p.count, p.groups, p.cost, blockIdx.x, a.split, status);
  } else {
    const PartArgs& p = a.part[1];
    decode_run<kNarrow>(t + p.first, p.count, p.groups, p.cost, blockIdx.x - a.split, gridDim.x - a.split, status);
  }
}

__global__ void __launch_bounds__(kThreads, 1) decode_table_kernel(const DevTensor* __restrict__ ts,
                                                                    const __grid_constant__ SplitArgs a,
                                                                    int32_t* status) {
  allow_dependents();
  wait_prerequisites();  // the descriptor table itself was copied in by earlier stream work
  decode_split(ts, a, status);
}

// Small batches travel inside the launch's parameter block.
template <int N>
struct InlineBatch {
  DevTensor t[N];
};
constexpr int kInlineMax = ECF8_BATCH_INLINE_MAX;

template <int N>
__global__ void __launch_bounds__(kThreads, 1) decode_inline_kernel(const __grid_constant__ InlineBatch<N> b,
                                                                     const __grid_constant__ SplitArgs a,
                                                                     int32_t* status) {
  allow_dependents();
  decode_split(b.t, a, status);
}

std::atomic<uint64_t> g_launches{0};

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
  const int bytes = (int)sizeof(Smem);
  const cudaFuncAttribute a = cudaFuncAttributeMaxDynamicSharedMemorySize;
  if (cudaFuncSetAttribute(decode_table_kernel, a, bytes) || cudaFuncSetAttribute(decode_inline_kernel<1>, a, bytes) ||
      cudaFuncSetAttribute(decode_inline_kernel<kInlineMax>, a, bytes))
    return ECF8_ERR_CUDA;
  int sms = 0, per_sm = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_inline_kernel<kInlineMax>, kThreads, bytes))
    return ECF8_ERR_CUDA;
  have = (uint32_t)(sms * (per_sm > 0 ? per_sm : 1));
  per_dev[dev].ctas.store(have);
  *ctas = have;
  return ECF8_OK;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

int check_info(const ecf8_info* info) {
  if (!info) return ECF8_ERR_ARG;
  Layout L;
  if (!compute_layout(info->n, info->code_bits, info->chunk_bytes, info->group_chunks, &L)) return ECF8_ERR_FORMAT;
  if (L.groups != info->n_groups || L.total != info->blob_bytes ||
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
  // the decoder's state machine needs a complete code (Kraft sum 1) or a
  // single value, which is what the encoder always writes
  int present = 0;
  for (int s = 0; s < 16; ++s) present += info->len[s] ? 1 : 0;
  if (info->n && present > 1 && kraft != (1ull << 16)) return ECF8_ERR_CODEBOOK;
  return ECF8_OK;
}

// The table width a tensor needs: wide when some code is 1 bit long.
int width_of(const ecf8_info* info) {
  for (int v = 0; v < 16; ++v)
    if (info->len[v] == 1) return kWide;
  return kNarrow;
}

// Estimated cost of decoding one group of a tensor, in units of about one
// decoded weight, fitted to per-CTA timings on B200: with the narrow table a
// group costs nearly the same whatever its code count (the walk over its 1 KB
// of stream dominates), with the wide table the weights it holds (8192 bits
// over the mean code length) add on top of the walk.  Only the split of work
// between CTAs depends on it, never the bytes decoded.
uint32_t group_cost(const ecf8_info* info) {
  const uint64_t bits = (uint64_t)kC * kT * 8;
  uint64_t codes = info->code_bits ? bits * info->n / info->code_bits : bits;
  if (codes > bits) codes = bits;
  return width_of(info) == kWide ? 3250u + (uint32_t)codes : 5200u + (uint32_t)codes / 10u;
}

DevTensor make_dev(const ecf8_info* info, const void* d_blob, uint8_t* d_out) {
  const uint8_t* b = static_cast<const uint8_t*>(d_blob);
  DevTensor t;
  t.cost_base = 0;
  t.gaps = reinterpret_cast<const uint32_t*>(b + info->gaps_off);
  t.groups = reinterpret_cast<const uint64_t*>(b + info->groups_off);
  t.stream = reinterpret_cast<const uint32_t*>(b + info->stream_off);
  t.nibbles = b + info->nibbles_off;
  t.out = d_out;
  t.n = info->n;
  t.code_bits = info->code_bits;
  t.n_groups = info->n_groups;
  t.group_base = 0;
  t.group_cost = group_cost(info);
  for (int s = 0; s < 16; ++s) t.len[s] = info->len[s];
  return t;
}

// Checks one tensor of a call; *skip is set for an empty tensor (n = 0),
// which the launch leaves out.
int check_tensor(const ecf8_tensor& t, bool* skip) {
  int rc = check_info(t.info);
  if (rc) return rc;
  if (t.info->chunk_bytes != (uint32_t)kC || t.info->group_chunks != (uint32_t)kT) return ECF8_ERR_UNSUPPORTED;
  *skip = t.info->n == 0;
  if (*skip) return ECF8_OK;
  if (!t.d_blob || !t.d_out || t.blob_size < t.info->blob_bytes) return ECF8_ERR_ARG;
  if (!aligned16(t.d_blob) || !aligned16(t.d_out)) return ECF8_ERR_ALIGN;
  return ECF8_OK;
}

// The descriptors of one launch: table[first, first + count), with the
// launch's group count and total estimated cost.
struct Part {
  int first = 0, count = 0;
  uint64_t groups = 0, cost = 0;
};

// Checks the tensors of a call and fills table[] with the descriptors of the
// non-empty ones: the wide-table ones first (part[0]), then the narrow ones
// (part[1]), each part with its own group and cost offsets.
int build_table(const ecf8_tensor* tensors, int count, DevTensor* table, Part part[2]) {
  part[0] = part[1] = Part();
  for (int i = 0; i < count; ++i) {
    bool skip = false;
    int rc = check_tensor(tensors[i], &skip);
    if (rc) return rc;
    if (!skip) part[width_of(tensors[i].info) == kWide ? 0 : 1].count++;
  }
  part[1].first = part[0].count;
  int at[2] = {0, part[1].first};
  for (int i = 0; i < count; ++i) {
    const ecf8_info* info = tensors[i].info;
    if (info->n == 0) continue;
    const int k = width_of(info) == kWide ? 0 : 1;
    DevTensor t = make_dev(info, tensors[i].d_blob, tensors[i].d_out);
    t.group_base = (uint32_t)part[k].groups;
    t.cost_base = part[k].cost;
    part[k].groups += t.n_groups;
    part[k].cost += kTensorSetupCost + (uint64_t)t.n_groups * t.group_cost;
    if (part[k].groups > 0xFFFFFFFFull) return ECF8_ERR_UNSUPPORTED;
    table[at[k]++] = t;
  }
  return ECF8_OK;
}

// One launch for both parts: the grid is split between them in proportion
// to their estimated cost.  Descriptors travel in the parameter block (h,
// when d_table is null) or are read from d_table (device, already filled).
int launch_parts(const DevTensor* h, const DevTensor* d_table, const Part part[2], int32_t* status,
                 cudaStream_t s, uint32_t max_ctas = 0) {
  const uint64_t groups = part[0].groups + part[1].groups;
  if (groups == 0) return ECF8_OK;
  uint32_t ctas = 0;
  int rc = grid_for_device(&ctas);
  if (rc) return rc;
  if (max_ctas && max_ctas < ctas) ctas = max_ctas;
  uint32_t grid = (uint32_t)(groups < ctas ? groups : ctas);
  // a launch with both parts needs a CTA for each (a cap of 1 is raised to 2)
  if (part[0].groups && part[1].groups && grid < 2) grid = 2;
  SplitArgs a;
  for (int k = 0; k < 2; ++k) a.part[k] = PartArgs{part[k].first, part[k].count, (uint32_t)part[k].groups, part[k].cost};
  if (part[0].groups == 0) {
    a.split = 0;
  } else if (part[1].groups == 0) {
    a.split = grid;
  } else {
    // of the two whole CTA counts nearest the cost share, the one whose
    // busier part finishes first
    const double cw = (double)part[0].cost, cn = (double)part[1].cost;
    const double f = cw / (cw + cn) * grid;
    uint32_t best = 1;
    double best_t = 0;
    for (uint32_t sp : {(uint32_t)f, (uint32_t)f + 1}) {
      sp = sp < 1 ? 1 : sp > grid - 1 ? grid - 1 : sp;
      const double t = cw / sp > cn / (grid - sp) ? cw / sp : cn / (grid - sp);
      if (best_t == 0 || t < best_t) {
        best = sp;
        best_t = t;
      }
    }
    a.split = best;
  }
  const int used = part[0].count + part[1].count;
  // every launch allows programmatic dependent launch (see wait_prerequisites)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = sizeof(Smem);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err;
  if (d_table) {
    err = cudaLaunchKernelEx(&cfg, decode_table_kernel, d_table, a, status);
  } else if (used == 1) {
    InlineBatch<1> b;
    b.t[0] = h[0];
    err = cudaLaunchKernelEx(&cfg, decode_inline_kernel<1>, b, a, status);
  } else {
    if (used > kInlineMax) return ECF8_ERR_ARG;
    InlineBatch<kInlineMax> b;
    for (int i = 0; i < used; ++i) b.t[i] = h[i];
    err = cudaLaunchKernelEx(&cfg, decode_inline_kernel<kInlineMax>, b, a, status);
  }
  if (err != cudaSuccess || cudaGetLastError() != cudaSuccess) return ECF8_ERR_CUDA;
  g_launches.fetch_add(1);
  return ECF8_OK;
}

}  // namespace
}  // namespace ecf8

namespace ecf8 {
void note_launch() { g_launches.fetch_add(1); }
}  // namespace ecf8

using namespace ecf8;

extern "C" {

int ecf8_layout_supported(uint32_t chunk_bytes, uint32_t group_chunks) {
  return chunk_bytes == (uint32_t)kC && group_chunks == (uint32_t)kT;
}

int ecf8_decode(const ecf8_info* info, const void* d_blob, size_t blob_size, uint8_t* d_out, size_t n,
                int32_t* d_status, cudaStream_t s) {
  if (!info) return ECF8_ERR_ARG;
  if (n != info->n) return ECF8_ERR_ARG;
  const ecf8_tensor one{info, d_blob, blob_size, d_out};
  DevTensor t[1];
  Part part[2];
  int rc = build_table(&one, 1, t, part);
  if (rc) return rc;
  return launch_parts(t, nullptr, part, d_status, s);
}

size_t ecf8_batched_workspace_size(int count) {
  return count > kInlineMax ? sizeof(DevTensor) * (size_t)count : 0;
}

int ecf8_decode_batched_ctas(const ecf8_tensor* tensors, int count, void* d_workspace, size_t workspace_bytes,
                             int32_t* d_status, cudaStream_t s, uint32_t max_ctas) {
  if (count < 0 || (count > 0 && !tensors)) return ECF8_ERR_ARG;
  if (count == 0) return ECF8_OK;
  if (count > kInlineMax) {
    if (!d_workspace || workspace_bytes < ecf8_batched_workspace_size(count)) return ECF8_ERR_WORKSPACE;
    if (!aligned16(d_workspace)) return ECF8_ERR_ALIGN;
  }
  std::vector<DevTensor> v((size_t)count);
  Part part[2];
  int rc = build_table(tensors, count, v.data(), part);
  if (rc) return rc;
  const size_t used = (size_t)part[0].count + (size_t)part[1].count;
  if (used == 0) return ECF8_OK;
  const DevTensor* d_table = nullptr;
  if (count > kInlineMax) {
    // the descriptor copy below reads a temporary host array, which a captured
    // graph would read again at replay, after the array is gone
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) return ECF8_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone) return ECF8_ERR_CAPTURE;
    if (cudaMemcpyAsync(d_workspace, v.data(), sizeof(DevTensor) * used, cudaMemcpyHostToDevice, s) != cudaSuccess)
      return ECF8_ERR_CUDA;
    d_table = static_cast<const DevTensor*>(d_workspace);
  }
  return launch_parts(v.data(), d_table, part, d_status, s, max_ctas);
}

int ecf8_decode_batched(const ecf8_tensor* tensors, int count, void* d_workspace, size_t workspace_bytes,
                        int32_t* d_status, cudaStream_t s) {
  return ecf8_decode_batched_ctas(tensors, count, d_workspace, workspace_bytes, d_status, s, 0);
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
  Part part[2];
  int rc = build_table(tensors, count, host_table, part);
  if (rc) return rc;
  const size_t used = (size_t)part[0].count + (size_t)part[1].count;
  if (used == 0) return ECF8_OK;
  DevTensor* table = nullptr;
  if ((rc = noalloc_table_address(&table))) return rc;
  if (cudaMemcpyAsync(table, host_table, sizeof(DevTensor) * used, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return ECF8_ERR_CUDA;
  return launch_parts(host_table, table, part, d_status, s);
}
