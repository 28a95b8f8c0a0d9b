// Library-internal constants and layout arithmetic for the ECF8 blob (version 3),
// shared by the host encoder (ecf8_host.cpp) and the decode kernels
// (ecf8_decode.cu).  The layout itself is documented in include/ecf8.h.
#pragma once

#include <stdint.h>

#include "ecf8.h"

namespace ecf8 {

constexpr uint32_t kMagic = 0x38464345u;  // "ECF8"
constexpr uint32_t kVersion = 3;
constexpr uint32_t kHeaderBytes = 128;
constexpr uint32_t kSectionAlign = 256;

struct Layout {
  uint64_t n, code_bits, groups;
  uint32_t C, T;
  uint64_t gaps_off, gaps_bytes;
  uint64_t groups_off, groups_bytes;
  uint64_t stream_off, stream_bytes;
  uint64_t nib_off, nib_bytes;
  uint64_t total;
};

inline uint64_t align_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

// Section sizes and offsets for n weights whose codes take code_bits bits.
inline bool compute_layout(uint64_t n, uint64_t code_bits, uint32_t C, uint32_t T, Layout* L) {
  if (C < 4 || C % 4 != 0 || T < 1) return false;
  L->n = n;
  L->code_bits = code_bits;
  L->C = C;
  L->T = T;
  const uint64_t group_bits = 8ull * C * T;
  L->groups = (code_bits + group_bits - 1) / group_bits;
  if (L->groups > 0xFFFFFFFFull) return false;
  const uint64_t chunks = L->groups * T;
  L->gaps_bytes = align_up((chunks + 7) / 8 * 4, 16);
  L->groups_bytes = 8 * (L->groups + 1);
  L->stream_bytes = n ? chunks * C + 16 : 0;
  L->nib_bytes = (n + 31) / 32 * 16;
  L->gaps_off = align_up(kHeaderBytes, kSectionAlign);
  L->groups_off = align_up(L->gaps_off + L->gaps_bytes, kSectionAlign);
  L->stream_off = align_up(L->groups_off + L->groups_bytes, kSectionAlign);
  L->nib_off = align_up(L->stream_off + L->stream_bytes, kSectionAlign);
  L->total = L->nib_off + L->nib_bytes;
  return true;
}

// Where the stream's word w (in reading order) is stored: inside each group
// of T chunks of C bytes the words are kept word-major, word m of chunk c at
// position m * T + c of the group, so that a warp reading word m of its T
// chunks reads adjacent words.
#if defined(__CUDACC__)
__host__ __device__
#endif
inline uint64_t stream_word_pos(uint64_t w, uint32_t C, uint32_t T) {
  const uint64_t per_chunk = C / 4, per_group = per_chunk * T;
  const uint64_t g = w / per_group, r = w % per_group;
  return g * per_group + (r % per_chunk) * T + r / per_chunk;
}

// The weight whose exponent is code i of the stream.  Codes follow the
// weights, except that inside every whole block of 8 weights they come in the
// order 0 4 1 5 2 6 3 7: a 32-bit word of 8 decoded exponents then holds
// weights 0-3 in the low nibbles of its bytes and weights 4-7 in the high
// ones.  A last block of fewer than 8 weights keeps weight order.
#if defined(__CUDACC__)
__host__ __device__
#endif
inline uint64_t coded_weight(uint64_t i, uint64_t n) {
  if ((i | 7) >= n) return i;
  return (i & ~7ull) | ((i & 7) >> 1) | ((i & 1) << 2);
}

// The stream position of weight k's code: the inverse of coded_weight.
#if defined(__CUDACC__)
__host__ __device__
#endif
inline uint64_t code_position(uint64_t k, uint64_t n) {
  if ((k | 7) >= n) return k;
  return (k & ~7ull) | ((k & 3) << 1) | ((k >> 2) & 1);
}

// Host side of the device encoder (ecf8_host.cpp): checks the codebook
// against the tensor's histogram and lays the blob out; writes the 128-byte
// header, the same as ecf8_encode does.
int prepare_blob(const ecf8_codebook* cb, const uint64_t hist[16], uint64_t n, uint32_t chunk_bytes,
                 uint32_t group_chunks, Layout* L, uint16_t code[16]);
void write_blob_prefix(uint8_t* blob, const Layout& L, const ecf8_codebook* cb, const uint16_t code[16]);

// Counts one kernel launch in ecf8_launch_count (ecf8_decode.cu).
void note_launch();

// What a decode kernel needs to know about one tensor, with device pointers
// already resolved into the blob's sections.
struct alignas(16) DevTensor {
  uint64_t cost_base;  // batched: estimated decode cost of all earlier tensors
  const uint32_t* gaps;
  const uint64_t* groups;
  const uint32_t* stream;
  const void* nibbles;  // 16-byte aligned
  uint8_t* out;
  uint64_t n;
  uint64_t code_bits;
  uint32_t n_groups;
  uint32_t group_base;  // batched: groups of all earlier tensors in the launch
  uint32_t group_cost;  // estimated decode cost of one group of this tensor
  uint8_t len[16];
};
static_assert(sizeof(DevTensor) == 96, "descriptor size is part of the workspace contract");

}  // namespace ecf8
