// GPU decoder of the BF16 variant (DFloat11 article §2-§3: the exponent
// field Huffman-coded per tensor over 256 values, sign and mantissa kept as
// one byte; blob layout as in bf16_oracle.c / ecf8_bf16_host.cpp).
//
// The same plan as the ECF8 decoder, with an 8-bit alphabet: one warp per
// group of 32 chunks of 32 stream bytes; each lane shifts its slice to its
// first code (the gap), zeroes the bits after its last code and walks its
// 272 bits a nibble (or a byte) at a time through a state machine over the
// code tree (one entry per (node, nibble or byte): the exponents whose codes
// end inside it, their count and the next node); zero-padding codes are
// subtracted by count; a warp scan
// places each lane's exponents; they are packed a byte each into lane-private
// shared memory, funnel-shifted into a byte stage, and 16 exponents plus 16
// kept bytes become 16 BF16 values per lane step.  The group's kept bytes are
// loaded into registers before its walk, so that their DRAM latency overlaps
// it; the next group's stream words are loaded before the current group is
// processed.  One launch covers up to ECF8_BF16_BATCH_MAX tensors of one
// layout: each persistent CTA takes a contiguous run of their groups and
// restages its table where the run crosses into the next tensor.  Launches
// allow programmatic dependent launch: a decode's CTAs may become resident
// while the previous kernel on the stream drains, and wait for it before they
// touch global memory.
//
// Four table layouts; the host picks wide, byte or narrow per tensor (the
// lane-private one only when asked for):
//  - wide: when a 1-bit code exists a nibble may end 4 codes; 64-bit entries
//    {exponents, next node << 7 | 8 count << 16}, as the host builds them;
//    a group may hold 8192 codes, so 13 warps fit an SM;
//  - narrow: shortest code >= 2 bits, so a nibble ends at most 2 codes and an
//    entry packs into 32 bits (exponents 0-15, node 16-23, 8 count 27-31); a
//    group holds at most 4096 codes and a lane 128, which halves the warp's
//    buffers, so 16 warps fit;
//  - narrow, lane-private: as narrow, with trees of at most 31 nodes copied
//    once per lane (entry i of lane l at word 32 i + l), so that each lane
//    reads its own bank and a lookup is one shared-memory wavefront;
//  - byte: shortest code >= 2 bits and at most 31 nodes: one entry per
//    (node, byte), composed on the device from two nibble entries (a byte
//    ends at most 4 codes: 64-bit entries {exponents, node << 11 | (node &
//    15) << 3 | 8 count << 24}, slots swizzled across the bank pairs), so a
//    lane walks 34 steps instead of 68 (the default for such codes).
// Corrupt input is reported through the status word; no access leaves its
// buffer and no loop runs without a bound.
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <string.h>

#include <type_traits>
#include <vector>

#include "ecf8.h"
#include "ecf8_format.h"

namespace ecf8_bf16 {
namespace {

constexpr int kC = 32, kT = 32;
constexpr int kWords = kC / 4;             // stream words per chunk
constexpr int kSpanBits = 8 * kC;          // 256
constexpr int kNibbles = 68;               // 272 bits: a lane may own up to 256 + 15 bits
constexpr int kPadBits = 4 * kNibbles;
constexpr int kKeep = 8;                   // kept-byte units per lane loaded before the walk

enum Layout { kWide = ECF8_BF16_LAYOUT_WIDE, kNarrow = ECF8_BF16_LAYOUT_NARROW,
              kNarrowLane = ECF8_BF16_LAYOUT_NARROW_LANE, kByte = ECF8_BF16_LAYOUT_BYTE };

template <int V>
struct Cfg {
  // codes a lane / a group can hold: shortest code 1 bit (wide) or >= 2 bits (the others)
  static constexpr int kLaneCodes = V == kWide ? 4 * (kNibbles + 1) : 128;
  static constexpr int kPrivWords = kLaneCodes / 4 + 1;
  static constexpr int kMaxCodes = V == kWide ? kSpanBits * kT : kSpanBits * kT / 2;
  static constexpr int kStageWords = (kMaxCodes + 32) / 4;  // 15 head bytes + codes, whole 16-byte units
  static constexpr int kMaxWarps = V == kWide ? 13 : 16;
};

template <int V>
struct alignas(16) WarpArea {
  uint32_t priv[Cfg<V>::kPrivWords * 32];  // word k of lane l at k*32 + l
  uint32_t stage[Cfg<V>::kStageWords];     // exponent byte i at byte i (from the group's 16-aligned base)
};

// One tensor of a launch.
struct Args {
  const uint32_t* gaps;
  const uint64_t* groups;
  const uint32_t* stream;
  const uint8_t* kept;
  uint16_t* out;
  const uint2* table;   // the host-built nibble table (device)
  uint64_t n, code_bits;
  uint32_t n_groups, lmin;
  uint32_t nodes;       // tree nodes; the error node is node `nodes`
  uint32_t group_base;  // groups of the launch's earlier tensors
};

// Up to ECF8_BF16_BATCH_MAX tensors of one table layout, in the launch's
// parameters; their groups are numbered consecutively in tensor order.
struct Batch {
  Args t[ECF8_BF16_BATCH_MAX];
  uint32_t count, total_groups;
  uint32_t zc_off, warp_off;  // shared-memory offsets: zero-code table, warp areas
};
static_assert(sizeof(Batch) <= 4096, "kernel parameter block");

// Checked builds (-DECF8_CHECKED, libecf8_checked.so) test each index a
// kernel reads or stores against its buffer; a failed test skips the access
// and sets ECF8_STATUS_BOUNDS.  Release builds compile the tests away.
#ifdef ECF8_CHECKED
__device__ __forceinline__ bool in_bounds(bool ok, int32_t* status) {
  if (!ok && status) atomicOr(status, ECF8_STATUS_BOUNDS);
  return ok;
}
#else
__device__ __forceinline__ bool in_bounds(bool, int32_t*) { return true; }
#endif

template <int V>
__host__ __device__ __forceinline__ uint32_t table_bytes(uint32_t nodes) {
  const uint32_t entries = (nodes + 1) * 16;
  return V == kWide ? entries * 8 : V == kNarrow ? entries * 4 : V == kNarrowLane ? entries * 128 : (nodes + 1) * 2048;
}

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

// Unit u of the group: 16 weights from base + 16u, their exponents at stage
// bytes 16u..16u+15.  Whole units take two 16-byte stores; the group's ragged
// first and last unit store only the weights inside the group, whose
// positions relative to base are [head, head + count).
template <int V>
__device__ __forceinline__ void emit_unit(uint16_t* out_base, uint64_t base, uint64_t n, const uint4* st,
                                          uint32_t head, uint32_t count, uint32_t u, uint4 kb, int32_t* status) {
  const uint4 ex = in_bounds(4 * u + 4 <= (uint32_t)Cfg<V>::kStageWords, status) ? st[u] : make_uint4(0, 0, 0, 0);
  const uint32_t e4[4] = {ex.x, ex.y, ex.z, ex.w}, k4[4] = {kb.x, kb.y, kb.z, kb.w};
  uint32_t o[8];
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    o[2 * w] = pair_bf16(__byte_perm(k4[w], 0u, 0x4140), __byte_perm(e4[w], 0u, 0x4140));
    o[2 * w + 1] = pair_bf16(__byte_perm(k4[w], 0u, 0x4342), __byte_perm(e4[w], 0u, 0x4342));
  }
  const uint32_t r0 = 16 * u;
  if (r0 >= head && r0 + 16 <= head + count) {
    if (in_bounds(base + r0 + 16 <= n, status)) {
      uint4* dst = reinterpret_cast<uint4*>(out_base + r0);
      dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
  } else {
#pragma unroll
    for (int k = 0; k < 16; ++k)
      if (r0 + k >= head && r0 + k < head + count && in_bounds(base + r0 + k < n, status))
        out_base[r0 + k] = (uint16_t)(o[k >> 1] >> (16 * (k & 1)));
  }
}

__device__ __forceinline__ uint32_t nibble_of(const uint32_t* sw, int j) {
  return (sw[j >> 3] >> (28 - 4 * (j & 7))) & 15u;
}

// One table step: the entry for the current node and the lane's next nibble
// (or byte); gives the exponents (first lowest) and 8 x their count.
template <int V>
struct Walker {
  // narrow entry: exponents bits 0-15, node bits 16-23, 8 x count bits 27-31
  static constexpr int kSteps = kNibbles;
  const uint8_t* table;
  uint32_t lane_term, limit;
  int32_t* status;
  uint32_t e = 0;
  __device__ __forceinline__ Walker(const uint8_t* t, uint32_t lane, uint32_t lim, int32_t* st)
      : table(t), lane_term(V == kNarrowLane ? lane * 4 : 0), limit(lim), status(st) {}
  __device__ __forceinline__ void step(const uint32_t* sw, int j, uint32_t& syms, uint32_t& bits8) {
    const uint32_t nib = nibble_of(sw, j);
    // lane-private: byte (node * 16 + nib) * 128 + lane * 4; shared: (node * 16 + nib) * 4
    uint32_t at = V == kNarrowLane ? (((e >> 5) & (0x1Fu << 11)) | (nib << 7) | lane_term)
                                   : (((e >> 10) & (0xFFu << 6)) | (nib << 2));
    if (!in_bounds(at + 4 <= limit, status)) at = 0;
    e = *reinterpret_cast<const uint32_t*>(table + at);
    syms = e & 0xFFFFu;
    bits8 = e >> 27;
  }
  __device__ __forceinline__ uint32_t node() const { return (e >> 16) & 0xFFu; }
};

template <>
struct Walker<kWide> {
  static constexpr int kSteps = kNibbles;
  const uint8_t* table;
  uint32_t limit;
  int32_t* status;
  uint32_t y = 0;
  __device__ __forceinline__ Walker(const uint8_t* t, uint32_t, uint32_t lim, int32_t* st)
      : table(t), limit(lim), status(st) {}
  __device__ __forceinline__ void step(const uint32_t* sw, int j, uint32_t& syms, uint32_t& bits8) {
    uint32_t at = (y & (0xFFu << 7)) | (nibble_of(sw, j) << 3);
    if (!in_bounds(at + 8 <= limit, status)) at = 0;
    const uint2 e = *reinterpret_cast<const uint2*>(table + at);
    y = e.y;
    syms = e.x;
    bits8 = e.y >> 16;
  }
  __device__ __forceinline__ uint32_t node() const { return (y >> 7) & 0xFFu; }
};

// Byte-table slot of (node, byte): the low 4 bits of the byte index are
// XORed with its high nibble and the node's low 4 bits (a bijection within the
// node's 256 entries), so that the 8-byte entries the lanes of a warp read
// spread over the bank pairs by the whole byte and node, not by the byte's low
// nibble alone.
__host__ __device__ __forceinline__ uint32_t byte_slot(uint32_t node, uint32_t byte) {
  return node * 256 + ((byte & 0xF0u) | ((byte ^ (byte >> 4) ^ node) & 15u));
}

template <>
struct Walker<kByte> {
  // entry (node, byte) at byte offset 8 * byte_slot(node, byte); y carries
  // node << 11 | (node & 15) << 3, so one LOP3 gives the next slot's offset
  static constexpr int kSteps = kNibbles / 2;
  const uint8_t* table;
  uint32_t limit;
  int32_t* status;
  uint32_t y = 0;
  __device__ __forceinline__ Walker(const uint8_t* t, uint32_t, uint32_t lim, int32_t* st)
      : table(t), limit(lim), status(st) {}
  __device__ __forceinline__ void step(const uint32_t* sw, int j, uint32_t& syms, uint32_t& bits8) {
    const uint32_t b8 = ((sw[j >> 2] >> (24 - 8 * (j & 3))) & 0xFFu) << 3;
    const uint32_t swz8 = b8 ^ ((b8 >> 4) & 0x78u);  // (byte & 0xF0 | (byte ^ byte >> 4) & 15) * 8
    uint32_t at = (y & ((0x1Fu << 11) | (15u << 3))) ^ swz8;
    if (!in_bounds(at + 8 <= limit, status)) at = 0;
    const uint2 e = *reinterpret_cast<const uint2*>(table + at);
    y = e.y;
    syms = e.x;
    bits8 = e.y >> 24;
  }
  __device__ __forceinline__ uint32_t node() const { return (y >> 11) & 0x1Fu; }
};

template <int V>
__device__ void process_group(const Args& a, uint32_t g, const GroupIn& in, const uint8_t* table,
                              const uint16_t* zero_codes, WarpArea<V>* wa, int32_t* status) {
  using C = Cfg<V>;
  const uint32_t lane = threadIdx.x & 31;
  const uint64_t off0 = in.off0, off1 = in.off1;
  const bool offsets_ok = off0 <= off1 && off1 <= a.n && off1 - off0 <= (uint64_t)C::kMaxCodes;

  // the group's kept bytes, in flight during the walk
  const uint64_t base = off0 & ~15ull;
  const uint32_t head = (uint32_t)(off0 & 15);
  const uint32_t count = offsets_ok ? (uint32_t)(off1 - off0) : 0u;
  // no kept byte is read for a group whose offsets fail their check
  const uint32_t units = offsets_ok ? (head + count + 15) >> 4 : 0u;
  const uint4* kept_units = reinterpret_cast<const uint4*>(a.kept + base);
  uint4 kp[kKeep];
#pragma unroll
  for (int i = 0; i < kKeep; ++i) {
    const uint32_t u = lane + 32 * i;
    kp[i] = u < units && in_bounds((base >> 4) + u < (a.n + 15) / 16, status) ? __ldg(kept_units + u)
                                                                              : make_uint4(0, 0, 0, 0);
  }

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

  // the nibble machine: 68 steps, exponents packed a byte each (codes past
  // the lane's capacity, which in a valid stream only the zero padding
  // produces, are counted but not stored)
  uint32_t* priv = wa->priv + lane;
  Walker<V> walk(table, lane, table_bytes<V>(a.nodes), status);
  uint32_t acc = 0, sh = 0, words = 0;
#pragma unroll
  for (int j = 0; j < Walker<V>::kSteps; ++j) {
    uint32_t syms, bits8;
    walk.step(sw, j, syms, bits8);
    acc |= syms << sh;
    const uint32_t carry = __funnelshift_l(syms, 0u, sh);
    sh += bits8;
    if (sh >= 32) {
      if (words < (uint32_t)C::kPrivWords) priv[32 * words] = acc;
      ++words;
      acc = carry;
      sh -= 32;
    }
  }
  if (sh && words < (uint32_t)C::kPrivWords) priv[32 * words] = acc;
  const uint32_t emitted = 4 * words + sh / 8;
  const uint32_t extra = zero_codes[kPadBits - (E < (uint32_t)kPadBits ? E : (uint32_t)kPadBits)];
  const bool bad = walk.node() == a.nodes || emitted < extra || emitted - extra > (uint32_t)C::kLaneCodes;
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

  // exponent bytes into the stage at byte head + start
  uint32_t* stage = wa->stage;
  const uint32_t q = head + start;
  const uint32_t d0 = q >> 2, dl = cnt ? (q + cnt - 1) >> 2 : 0;
  constexpr uint32_t kSW = (uint32_t)C::kStageWords, kPW = (uint32_t)C::kPrivWords;
  if (cnt && in_bounds(dl < kSW, status)) {
    stage[d0] = 0;
    stage[dl] = 0;
  }
  __syncwarp();
  if (cnt) {
    const uint32_t r = (q & 3) * 8;
    const uint32_t used = (cnt + 3) / 4;
    if ((cnt & 3) && in_bounds(used - 1 < kPW, status)) priv[32 * (used - 1)] &= (1u << (8 * (cnt & 3))) - 1;
    const uint32_t nwd = dl - d0 + 1;
    uint32_t prev = priv[0];
    if (in_bounds(d0 < kSW, status)) atomicOr(&stage[d0], prev << r);
    uint32_t j = 1;
#pragma unroll 4
    for (; j + 1 < nwd; ++j) {
      const uint32_t cur = in_bounds(j < kPW, status) ? priv[32 * j] : 0u;
      if (in_bounds(d0 + j < kSW, status)) stage[d0 + j] = __funnelshift_l(prev, cur, r);
      prev = cur;
    }
    if (nwd > 1) {
      const uint32_t cur = j < used && in_bounds(j < kPW, status) ? priv[32 * j] : 0;
      if (in_bounds(d0 + j < kSW, status)) atomicOr(&stage[d0 + j], __funnelshift_l(prev, cur, r));
    }
  }
  __syncwarp();

  // 16 weights per lane step: 16 exponent bytes + 16 kept bytes -> 32 output bytes
  const uint4* st = reinterpret_cast<const uint4*>(stage);
  uint16_t* out_base = a.out + base;
#pragma unroll
  for (int i = 0; i < kKeep; ++i) {
    const uint32_t u = lane + 32 * i;
    if (u < units) emit_unit<V>(out_base, base, a.n, st, head, count, u, kp[i], status);
  }
  for (uint32_t u = lane + 32 * kKeep; u < units; u += 32) {
    const uint4 kb = in_bounds((base >> 4) + u < (a.n + 15) / 16, status) ? __ldg(kept_units + u)
                                                                           : make_uint4(0, 0, 0, 0);
    emit_unit<V>(out_base, base, a.n, st, head, count, u, kb, status);
  }
  __syncwarp();
}

// The host's 64-bit entry {exponents, next node << 7 | 8 count << 16} in the
// narrow 32-bit form (the host picks a narrow layout only when no entry holds
// more than two exponents).
__device__ __forceinline__ uint32_t narrow_entry(uint2 w) {
  return (w.x & 0xFFFFu) | (((w.y >> 7) & 0xFFu) << 16) | (((w.y >> 16) & 0x1Fu) << 27);
}

// Tensor a's decode table and zero-code counts into shared memory (every
// thread of the CTA takes part; the first warp area serves as scratch).
template <int V>
__device__ __forceinline__ void stage_table(const Args& a, uint8_t* smem, uint32_t zc_off, uint32_t warp_off) {
  const uint32_t entries = (a.nodes + 1) * 16;
  const uint2* src = a.table;
  if (V == kWide) {
    uint2* t = reinterpret_cast<uint2*>(smem);
#pragma unroll 8
    for (uint32_t i = threadIdx.x; i < entries; i += blockDim.x) t[i] = __ldg(src + i);
  } else if (V == kNarrow) {
    uint32_t* t = reinterpret_cast<uint32_t*>(smem);
#pragma unroll 8
    for (uint32_t i = threadIdx.x; i < entries; i += blockDim.x) t[i] = narrow_entry(__ldg(src + i));
  } else if (V == kByte) {
    // the nibble entries once into scratch, then two of them per (node, byte)
    uint2* once = reinterpret_cast<uint2*>(smem + warp_off);
    for (uint32_t i = threadIdx.x; i < entries; i += blockDim.x) once[i] = __ldg(src + i);
    __syncthreads();
    uint2* t = reinterpret_cast<uint2*>(smem);
    for (uint32_t i = threadIdx.x; i < (a.nodes + 1) * 256; i += blockDim.x) {
      const uint32_t node = i >> 8, byte = i & 255;
      const uint2 e1 = once[node * 16 + (byte >> 4)];
      const uint32_t n1 = (e1.y >> 7) & 0xFFu, c1 = (e1.y >> 16) & 0x3Fu;
      const uint2 e2 = once[(n1 <= a.nodes ? n1 : a.nodes) * 16 + (byte & 15)];
      const uint32_t n2 = n1 == a.nodes ? a.nodes : (e2.y >> 7) & 0xFFu, c2 = (e2.y >> 16) & 0x3Fu;
      t[byte_slot(node, byte)] =
          make_uint2(e1.x | (c1 < 32 ? e2.x << c1 : 0u), (n2 << 11) | ((n2 & 15u) << 3) | ((c1 + c2) << 24));
    }
  } else {
    // each entry read once into scratch, then copied to every lane's slot
    uint32_t* once = reinterpret_cast<uint32_t*>(smem + warp_off);
    for (uint32_t i = threadIdx.x; i < entries; i += blockDim.x) once[i] = narrow_entry(__ldg(src + i));
    __syncthreads();
    uint32_t* t = reinterpret_cast<uint32_t*>(smem);
    for (uint32_t i = threadIdx.x; i < entries * 32; i += blockDim.x) t[i] = once[i >> 5];
  }
  uint16_t* zero_codes = reinterpret_cast<uint16_t*>(smem + zc_off);
  for (int z = threadIdx.x; z <= kPadBits; z += blockDim.x) zero_codes[z] = (uint16_t)(z / a.lmin);
}

// Persistent CTAs, each over a contiguous run of the batch's groups.  The run
// is cut at tensor boundaries into segments; for each segment the CTA stages
// that tensor's table, then its warps take the segment's groups in turn, each
// fetching its next group's stream slice while it decodes the current one.
template <int V>
__global__ void __launch_bounds__(Cfg<V>::kMaxWarps * 32, 1)
    decode_kernel(const __grid_constant__ Batch b, int32_t* status) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  // programmatic dependent launch: the next kernel on the stream may start
  // its CTAs early; this one touches no global memory (blobs, tables or
  // outputs the previous kernel may still use) before that kernel completes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const uint32_t warps = blockDim.x >> 5, warp = threadIdx.x >> 5;
  const uint32_t g_begin = (uint32_t)((uint64_t)b.total_groups * blockIdx.x / gridDim.x);
  const uint32_t g_end = (uint32_t)((uint64_t)b.total_groups * (blockIdx.x + 1) / gridDim.x);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const uint16_t* zero_codes = reinterpret_cast<const uint16_t*>(smem_raw + b.zc_off);
  WarpArea<V>* wa = reinterpret_cast<WarpArea<V>*>(smem_raw + b.warp_off) + warp;
  uint32_t k = 0;
  for (uint32_t seg = g_begin; seg < g_end;) {
    while (k + 1 < b.count && b.t[k + 1].group_base <= seg) ++k;
    const Args& a = b.t[k];
    const uint32_t seg_end = min(g_end, a.group_base + a.n_groups);
    uint32_t g = seg + warp;
    GroupIn in;
    if (g < seg_end) fetch_group(a, g - a.group_base, in);  // in flight while the table is staged
    __syncthreads();  // the previous segment's warps are done with the table
    stage_table<V>(a, smem_raw, b.zc_off, b.warp_off);
    __syncthreads();
    for (; g < seg_end; g += warps) {
      GroupIn nx;
      const uint32_t gn = g + warps;
      const bool more = gn < seg_end;
      if (more) fetch_group(a, gn - a.group_base, nx);
      process_group<V>(a, g - a.group_base, in, smem_raw, zero_codes, wa, status);
      if (more) in = nx;
    }
    seg = seg_end;
  }
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }
uint32_t up16(uint32_t x) { return (x + 15) & ~15u; }

// One launch over ts[0, count) (count <= ECF8_BF16_BATCH_MAX, every tensor
// non-empty and holdable by layout V).
template <int V>
int launch(const Args* ts, uint32_t count, int32_t* d_status, cudaStream_t s) {
  Batch b;
  memset(&b, 0, sizeof(b));
  uint64_t total = 0;
  uint32_t tbytes = 0;
  for (uint32_t i = 0; i < count; ++i) {
    b.t[i] = ts[i];
    b.t[i].group_base = (uint32_t)total;
    total += ts[i].n_groups;
    const uint32_t tb = table_bytes<V>(ts[i].nodes);
    tbytes = tb > tbytes ? tb : tbytes;
  }
  if (total == 0) return ECF8_OK;
  if (total > 0xFFFFFFFFull) return ECF8_ERR_ARG;
  b.count = count;
  b.total_groups = (uint32_t)total;
  b.zc_off = tbytes;
  b.warp_off = up16(b.zc_off + 2 * (kPadBits + 1));
  int dev = 0, sms = 0, smem_max = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) ||
      cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev))
    return ECF8_ERR_CUDA;
  if ((uint32_t)smem_max <= b.warp_off) return ECF8_ERR_UNSUPPORTED;
  const uint32_t fit = ((uint32_t)smem_max - b.warp_off) / (uint32_t)sizeof(WarpArea<V>);
  const uint32_t warps = fit < (uint32_t)Cfg<V>::kMaxWarps ? fit : (uint32_t)Cfg<V>::kMaxWarps;
  if (warps == 0) return ECF8_ERR_UNSUPPORTED;
  const uint32_t smem = b.warp_off + warps * (uint32_t)sizeof(WarpArea<V>);
  if (cudaFuncSetAttribute(decode_kernel<V>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_max))
    return ECF8_ERR_CUDA;
  const uint64_t ctas_needed = (total + warps - 1) / warps;
  const uint32_t grid = (uint32_t)(ctas_needed < (uint64_t)sms ? ctas_needed : (uint64_t)sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(warps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, decode_kernel<V>, b, d_status) != cudaSuccess || cudaGetLastError() != cudaSuccess)
    return ECF8_ERR_CUDA;
  ecf8::note_launch();
  return ECF8_OK;
}

int launch_layout(int layout, const Args* ts, uint32_t count, int32_t* d_status, cudaStream_t s) {
  switch (layout) {
    case kWide: return launch<kWide>(ts, count, d_status, s);
    case kNarrow: return launch<kNarrow>(ts, count, d_status, s);
    case kNarrowLane: return launch<kNarrowLane>(ts, count, d_status, s);
    default: return launch<kByte>(ts, count, d_status, s);
  }
}

}  // namespace
}  // namespace ecf8_bf16

using namespace ecf8_bf16;

namespace ecf8_bf16 {
namespace {

uint32_t shortest(const ecf8_bf16_info* info) {
  uint32_t lmin = 16;
  for (int v = 0; v < 256; ++v)
    if (info->len[v] && info->len[v] < lmin) lmin = info->len[v];
  return lmin;
}

bool layout_holds(int layout, uint32_t lmin, uint32_t nodes) {
  switch (layout) {
    case kWide: return true;
    case kNarrow: return lmin >= 2;
    case kNarrowLane:
    case kByte: return lmin >= 2 && nodes + 1 <= 32;
    default: return false;
  }
}

}  // namespace
}  // namespace ecf8_bf16

extern "C" int ecf8_bf16_auto_layout(const ecf8_bf16_info* info) {
  if (!info) return ECF8_ERR_ARG;
  const uint32_t nodes = ecf8_bf16_table_nodes(info);
  if (nodes == 0) return ECF8_ERR_CODEBOOK;
  const uint32_t lmin = shortest(info);
  if (lmin == 1) return kWide;
  return nodes + 1 <= 32 ? kByte : kNarrow;
}

namespace ecf8_bf16 {
namespace {

// Checks one tensor and fills its launch arguments; resolves AUTO.
int prepare(const ecf8_bf16_tensor& t, int* layout, Args* a) {
  const ecf8_bf16_info* info = t.info;
  if (!info) return ECF8_ERR_ARG;
  if (info->chunk_bytes != (uint32_t)kC || info->group_chunks != (uint32_t)kT) return ECF8_ERR_UNSUPPORTED;
  if (info->n == 0) return ECF8_OK;
  if (!t.d_blob || !t.d_table || !t.d_out) return ECF8_ERR_ARG;
  if (!aligned16(t.d_blob) || !aligned16(t.d_table) || !aligned16(t.d_out)) return ECF8_ERR_ALIGN;
  const uint32_t nodes = ecf8_bf16_table_nodes(info);
  if (nodes == 0) return ECF8_ERR_CODEBOOK;
  const uint32_t lmin = shortest(info);
  if (*layout == ECF8_BF16_LAYOUT_AUTO) *layout = lmin == 1 ? kWide : nodes + 1 <= 32 ? kByte : kNarrow;
  if (!layout_holds(*layout, lmin, nodes)) return ECF8_ERR_UNSUPPORTED;
  const uint8_t* b = static_cast<const uint8_t*>(t.d_blob);
  a->gaps = reinterpret_cast<const uint32_t*>(b + info->gaps_off);
  a->groups = reinterpret_cast<const uint64_t*>(b + info->groups_off);
  a->stream = reinterpret_cast<const uint32_t*>(b + info->stream_off);
  a->kept = b + info->kept_off;
  a->out = t.d_out;
  a->table = static_cast<const uint2*>(t.d_table);
  a->n = info->n;
  a->code_bits = info->code_bits;
  a->n_groups = info->n_groups;
  a->lmin = lmin;
  a->nodes = nodes;
  a->group_base = 0;
  return ECF8_OK;
}

}  // namespace
}  // namespace ecf8_bf16

extern "C" int ecf8_bf16_decode_layout(const ecf8_bf16_info* info, const void* d_blob, const void* d_table,
                                       uint16_t* d_out, size_t n, int32_t* d_status, cudaStream_t s, int layout) {
  if (!info || n != info->n) return ECF8_ERR_ARG;
  if (layout < ECF8_BF16_LAYOUT_AUTO || layout > ECF8_BF16_LAYOUT_BYTE) return ECF8_ERR_ARG;
  const ecf8_bf16_tensor t = {info, d_blob, d_table, d_out};
  Args a;
  const int rc = prepare(t, &layout, &a);
  if (rc != ECF8_OK || n == 0) return rc;
  return launch_layout(layout, &a, 1, d_status, s);
}

extern "C" int ecf8_bf16_decode(const ecf8_bf16_info* info, const void* d_blob, const void* d_table, uint16_t* d_out,
                                size_t n, int32_t* d_status, cudaStream_t s) {
  return ecf8_bf16_decode_layout(info, d_blob, d_table, d_out, n, d_status, s, ECF8_BF16_LAYOUT_AUTO);
}

extern "C" int ecf8_bf16_decode_batched(const ecf8_bf16_tensor* tensors, int count, int32_t* d_status,
                                        cudaStream_t s) {
  if (count < 0 || (count > 0 && !tensors)) return ECF8_ERR_ARG;
  // every tensor checked before anything is enqueued
  std::vector<Args> by_layout[4];
  for (int i = 0; i < count; ++i) {
    int layout = ECF8_BF16_LAYOUT_AUTO;
    Args a;
    const int rc = prepare(tensors[i], &layout, &a);
    if (rc != ECF8_OK) return rc;
    if (tensors[i].info->n) by_layout[layout].push_back(a);
  }
  for (int l = 0; l < 4; ++l)
    for (size_t i = 0; i < by_layout[l].size(); i += ECF8_BF16_BATCH_MAX) {
      const size_t c = by_layout[l].size() - i < (size_t)ECF8_BF16_BATCH_MAX ? by_layout[l].size() - i
                                                                              : (size_t)ECF8_BF16_BATCH_MAX;
      const int rc = launch_layout(l, by_layout[l].data() + i, (uint32_t)c, d_status, s);
      if (rc != ECF8_OK) return rc;
    }
  return ECF8_OK;
}
