// ECF8 encoder on the GPU: the same blob as the host encoder, byte for byte.
//
// The ECF8 walkthrough encodes per tensor in order: exponent histogram
// (§3.1.1 step 1), Huffman code (step 2), canonical code table, bit-packed
// code stream with per-chunk gaps and per-group offsets (§3.2.1), raw sign
// and mantissa nibbles.  Here the histogram and every
// per-weight step run on the GPU; only the 16-symbol code construction and
// the 128-byte header stay on the host.  Steps:
//   histogram_kernel   exponent counts (16 per tensor)
//   seg_bits_kernel    code bits of every 4096-weight segment
//   scan_kernel        segment start bits (exclusive scan, one CTA)
//   pack_kernel        the code stream (codes of each whole 8-weight block in
//                      the order 0 4 1 5 2 6 3 7, words word-major inside
//                      each group), gaps and group offsets
//   tail_kernel        offsets of groups that start past the stream end
//   nibble_kernel      8 signs and mantissas per 32-bit word
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <vector>

#include "ecf8.h"
#include "ecf8_format.h"

namespace ecf8 {
namespace {

constexpr int kSegThreads = 256;
constexpr int kPerThread = 16;                       // weights per thread: one 16-byte load
constexpr int kSeg = kSegThreads * kPerThread;       // weights per segment
constexpr int kScanThreads = 1024;

struct Code {
  uint8_t len[16];
  uint16_t code[16];
};

__device__ __forceinline__ uint32_t exponent_of(uint32_t b) { return (b >> 3) & 15u; }

// The 16 bytes of thread t's weights (zero past n).
__device__ __forceinline__ void load16(const uint8_t* x, uint64_t n, uint64_t i0, uint8_t b[16]) {
  if (i0 + 16 <= n) {
    const uint4 v = *reinterpret_cast<const uint4*>(x + i0);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 16; ++k) b[k] = (uint8_t)(w[k >> 2] >> (8 * (k & 3)));
  } else {
#pragma unroll
    for (int k = 0; k < 16; ++k) b[k] = i0 + k < n ? x[i0 + k] : 0;
  }
}

__global__ void histogram_kernel(const uint8_t* __restrict__ x, uint64_t n, unsigned long long* hist) {
  __shared__ unsigned int h[32][16];  // one row per warp
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < 32 * 16; i += blockDim.x) (&h[0][0])[i] = 0;
  __syncthreads();
  const uint64_t words = n / 16;
  const uint4* x4 = reinterpret_cast<const uint4*>(x);
  for (uint64_t w = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; w < words; w += (uint64_t)gridDim.x * blockDim.x) {
    const uint4 v = x4[w];
    const uint32_t q[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 16; ++k) atomicAdd(&h[warp][exponent_of(q[k >> 2] >> (8 * (k & 3)))], 1u);
  }
  if (blockIdx.x == 0)
    for (uint64_t i = words * 16 + threadIdx.x; i < n; i += blockDim.x) atomicAdd(&h[warp][exponent_of(x[i])], 1u);
  __syncthreads();
  if (threadIdx.x < 16) {
    unsigned long long s = 0;
    for (int r = 0; r < 32; ++r) s += h[r][threadIdx.x];
    if (s) atomicAdd(&hist[threadIdx.x], s);
  }
}

// Inclusive sum over the CTA (kSegThreads threads); *total gets the CTA's sum.
__device__ __forceinline__ uint32_t cta_inclusive_sum(uint32_t v, uint32_t* total) {
  __shared__ uint32_t warp_sums[kSegThreads / 32];
  const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, v, o);
    if (lane >= (uint32_t)o) v += t;
  }
  if (lane == 31) warp_sums[warp] = v;
  __syncthreads();
  uint32_t before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kSegThreads / 32; ++w) {
    const uint32_t s = warp_sums[w];
    before += (uint32_t)w < warp ? s : 0u;
    all += s;
  }
  __syncthreads();  // warp_sums is reused by the next call
  *total = all;
  return v + before;
}

__global__ void __launch_bounds__(kSegThreads) seg_bits_kernel(const uint8_t* __restrict__ x, uint64_t n, Code c,
                                                               uint32_t* seg_bits) {
  uint8_t b[16];
  load16(x, n, (uint64_t)blockIdx.x * kSeg + (uint64_t)threadIdx.x * kPerThread, b);
  const uint64_t i0 = (uint64_t)blockIdx.x * kSeg + (uint64_t)threadIdx.x * kPerThread;
  uint32_t bits = 0;
#pragma unroll
  for (int k = 0; k < 16; ++k) bits += i0 + k < n ? c.len[exponent_of(b[k])] : 0u;
  uint32_t total;
  cta_inclusive_sum(bits, &total);
  if (threadIdx.x == 0) seg_bits[blockIdx.x] = total;
}

// Exclusive scan of seg_bits[0, segs) into seg_start, by one CTA: each thread
// sums a contiguous run of segments, the CTA scans those sums, each thread
// then walks its run again.
__global__ void __launch_bounds__(kScanThreads) scan_kernel(const uint32_t* seg_bits, uint64_t segs,
                                                            uint64_t* seg_start) {
  __shared__ unsigned long long part[kScanThreads];
  const uint64_t per = (segs + kScanThreads - 1) / kScanThreads;
  const uint64_t a = threadIdx.x * per, e = a + per < segs ? a + per : segs;
  unsigned long long s = 0;
  for (uint64_t i = a; i < e; ++i) s += seg_bits[i];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int o = 1; o < kScanThreads; o <<= 1) {  // Hillis-Steele over the thread sums
    const unsigned long long t = threadIdx.x >= (unsigned)o ? part[threadIdx.x - o] : 0ull;
    __syncthreads();
    part[threadIdx.x] += t;
    __syncthreads();
  }
  unsigned long long run = part[threadIdx.x] - s;
  for (uint64_t i = a; i < e; ++i) {
    seg_start[i] = run;
    run += seg_bits[i];
  }
}

struct PackArgs {
  uint64_t n, code_bits, chunks, chunk_bits;
  uint32_t C, T;
  uint32_t* stream;
  uint32_t* gaps;
  uint64_t* offs;
};

// Chunk c (stream bits [c*chunk_bits, ...)) whose first code start is `pos`,
// that code being weight i (i = n: the stream end).
__device__ __forceinline__ void put_chunk(const PackArgs& p, uint64_t c, uint64_t pos, uint64_t i) {
  if (c >= p.chunks) return;
  const uint32_t gap = (uint32_t)(pos - c * p.chunk_bits);  // < 16: codes are at most 16 bits
  if (gap) atomicOr(&p.gaps[c / 8], gap << (4 * (c % 8)));
  if (c % p.T == 0) p.offs[c / p.T] = i;
}

__global__ void __launch_bounds__(kSegThreads) pack_kernel(const uint8_t* __restrict__ x, Code c,
                                                           const uint64_t* seg_start, PackArgs p) {
  uint8_t w[16];
  const uint64_t i0 = (uint64_t)blockIdx.x * kSeg + (uint64_t)threadIdx.x * kPerThread;
  load16(x, p.n, i0, w);
  // this thread's codes i0 .. i0+15 in stream order: code i0+k is weight
  // coded_weight(i0+k), one of the thread's own 16 weights
  uint8_t b[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const int r = k & 7, perm = (k & 8) | (r >> 1) | ((r & 1) << 2);
    b[k] = ((i0 + (k | 7)) < p.n) ? w[perm] : w[k];
  }
  uint32_t bits = 0;
#pragma unroll
  for (int k = 0; k < 16; ++k) bits += i0 + k < p.n ? c.len[exponent_of(b[k])] : 0u;
  uint32_t total;
  const uint32_t incl = cta_inclusive_sum(bits, &total);
  uint64_t pos = seg_start[blockIdx.x] + incl - bits;  // this thread's first code start
  if (i0 >= p.n) return;
  // start of the previous code (-1 before code 0); code i0-1 ends a whole
  // block, whose last code is its own last weight
  int64_t prev = -1;
  if (i0 > 0) prev = (int64_t)pos - (int64_t)c.len[exponent_of(x[i0 - 1])];
  // pack: MSB first within little-endian 32-bit words
  uint64_t word = pos / 32;
  const uint64_t first_word = word;
  uint64_t acc = 0;
  uint32_t nacc = (uint32_t)(pos % 32);  // bits of this word owned by earlier codes stay zero
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const uint64_t i = i0 + k;
    if (i >= p.n) break;
    const uint32_t e = exponent_of(b[k]);
    // the first chunk starting in (prev, pos] has this code first
    const uint64_t ch = pos / p.chunk_bits;
    if ((int64_t)(ch * p.chunk_bits) > prev) put_chunk(p, ch, pos, i);
    const uint32_t l = c.len[e];
    acc = (acc << l) | c.code[e];
    nacc += l;
    prev = (int64_t)pos;
    pos += l;
    if (nacc >= 32) {
      nacc -= 32;
      const uint32_t v = (uint32_t)(acc >> nacc);
      const uint64_t at = stream_word_pos(word, p.C, p.T);
      if (word == first_word) atomicOr(&p.stream[at], v);
      else p.stream[at] = v;
      ++word;
    }
  }
  if (nacc) atomicOr(&p.stream[stream_word_pos(word, p.C, p.T)], (uint32_t)(acc << (32 - nacc)));  // shared with the next thread
  // the stream end counts as a code start: chunks starting in (last start, end]
  if (i0 + 16 >= p.n) {
    const uint64_t c0 = ((uint64_t)(prev + 1) + p.chunk_bits - 1) / p.chunk_bits;  // first chunk start > prev
    for (uint64_t cc = c0; cc * p.chunk_bits <= pos && cc < p.chunks; ++cc) put_chunk(p, cc, pos, p.n);
  }
}

// Groups whose first chunk starts after the stream end begin at n, and so
// does the sentinel offs[groups].
__global__ void tail_kernel(PackArgs p, uint64_t groups) {
  const uint64_t first_past = (p.code_bits / p.chunk_bits) + 1;  // chunks starting after the end
  for (uint64_t g = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; g <= groups; g += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t c = g * p.T;
    if (g == groups || c >= first_past) p.offs[g] = p.n;
  }
}

// Signs and mantissas of 8 weights per word: byte k = weight k's sign (bit
// 7) and mantissa (bits 0-2), weight 4+k's mantissa (bits 4-6) and weight
// 4+((k+3)%4)'s sign (bit 3).  Given the two little-endian words of the 8
// bytes: a = weights 0-3, b = weights 4-7.
__device__ __forceinline__ uint32_t nibble_word(uint32_t a, uint32_t b) {
  const uint32_t rot = __funnelshift_l(b, b, 4);  // weight 4+k's sign to bit 3 of byte k+1 (mod 4)
  return (a & 0x87878787u) | ((b << 4) & 0x70707070u) | (rot & 0x08080808u);
}

__global__ void nibble_kernel(const uint8_t* __restrict__ x, uint64_t n, uint32_t* nib, uint64_t words) {
  for (uint64_t w = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; w < words; w += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t i = w * 8;
    uint2 q;
    if (i + 8 <= n) {
      q = *reinterpret_cast<const uint2*>(x + i);
    } else {
      uint32_t v[2] = {0, 0};
      for (int k = 0; k < 8 && i + k < n; ++k) v[k >> 2] |= (uint32_t)x[i + k] << (8 * (k & 3));
      q = make_uint2(v[0], v[1]);
    }
    nib[w] = nibble_word(q.x, q.y);
  }
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

int sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                 cudaSuccess)
    return 0;
  return sms;
}

}  // namespace
}  // namespace ecf8

using namespace ecf8;

extern "C" {

int ecf8_histogram_device(const uint8_t* d_fp8, size_t n, uint64_t* d_hist, cudaStream_t s) {
  if (!d_hist || (!d_fp8 && n)) return ECF8_ERR_ARG;
  if (!aligned16(d_fp8) || !aligned16(d_hist)) return ECF8_ERR_ALIGN;
  if (cudaMemsetAsync(d_hist, 0, 16 * sizeof(uint64_t), s) != cudaSuccess) return ECF8_ERR_CUDA;
  if (n == 0) return ECF8_OK;
  const int sms = sm_count();
  if (!sms) return ECF8_ERR_CUDA;
  const uint64_t words = n / 16;
  uint64_t want = (words + 255) / 256;
  const uint32_t grid = (uint32_t)(want < 1 ? 1 : want > (uint64_t)sms * 8 ? (uint64_t)sms * 8 : want);
  histogram_kernel<<<grid, 256, 0, s>>>(d_fp8, n, reinterpret_cast<unsigned long long*>(d_hist));
  return cudaGetLastError() == cudaSuccess ? ECF8_OK : ECF8_ERR_CUDA;
}

size_t ecf8_encode_device_workspace_size(size_t n) {
  const uint64_t segs = (n + kSeg - 1) / kSeg;
  return (size_t)(segs * (sizeof(uint32_t) + sizeof(uint64_t)) + 16);
}

int ecf8_encode_device(const uint8_t* d_fp8, size_t n, const uint64_t hist[16], const ecf8_codebook* cb,
                       uint32_t chunk_bytes, uint32_t group_chunks, void* d_blob, size_t blob_cap,
                       size_t* blob_bytes, void* d_workspace, size_t workspace_bytes, cudaStream_t s) {
  if (!blob_bytes || !d_blob || (!d_fp8 && n)) return ECF8_ERR_ARG;
  if (!aligned16(d_fp8) || !aligned16(d_blob)) return ECF8_ERR_ALIGN;
  Layout L;
  uint16_t code[16];
  int rc = prepare_blob(cb, hist, n, chunk_bytes, group_chunks, &L, code);
  if (rc) return rc;
  if (8ull * chunk_bytes < 16) return ECF8_ERR_ARG;  // a chunk must be longer than the longest code
  if (blob_cap < L.total) return ECF8_ERR_CAPACITY;
  const uint64_t segs = (n + kSeg - 1) / kSeg;
  if (n && (!d_workspace || workspace_bytes < ecf8_encode_device_workspace_size(n))) return ECF8_ERR_WORKSPACE;
  if (n && !aligned16(d_workspace)) return ECF8_ERR_ALIGN;
  uint8_t* blob = static_cast<uint8_t*>(d_blob);
  // the header from the host (a pageable copy: the host buffer has been read
  // when cudaMemcpyAsync returns), zeros up to the nibbles
  std::vector<uint8_t> prefix((size_t)kHeaderBytes);
  write_blob_prefix(prefix.data(), L, cb, code);
  if (cudaMemcpyAsync(blob, prefix.data(), prefix.size(), cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemsetAsync(blob + kHeaderBytes, 0, L.nib_off - kHeaderBytes, s) != cudaSuccess)
    return ECF8_ERR_CUDA;
  if (n) {
    Code c;
    for (int k = 0; k < 16; ++k) {
      c.len[k] = cb->len[k];
      c.code[k] = code[k];
    }
    uint64_t* seg_start = static_cast<uint64_t*>(d_workspace);
    uint32_t* seg_bits = reinterpret_cast<uint32_t*>(seg_start + segs);
    seg_bits_kernel<<<(uint32_t)segs, kSegThreads, 0, s>>>(d_fp8, n, c, seg_bits);
    scan_kernel<<<1, kScanThreads, 0, s>>>(seg_bits, segs, seg_start);
    PackArgs p;
    p.n = n;
    p.code_bits = L.code_bits;
    p.chunks = L.groups * group_chunks;
    p.chunk_bits = 8ull * chunk_bytes;
    p.C = chunk_bytes;
    p.T = group_chunks;
    p.stream = reinterpret_cast<uint32_t*>(blob + L.stream_off);
    p.gaps = reinterpret_cast<uint32_t*>(blob + L.gaps_off);
    p.offs = reinterpret_cast<uint64_t*>(blob + L.groups_off);
    pack_kernel<<<(uint32_t)segs, kSegThreads, 0, s>>>(d_fp8, c, seg_start, p);
    const int sms = sm_count();
    tail_kernel<<<(uint32_t)(sms ? sms : 1), 256, 0, s>>>(p, L.groups);
    const uint64_t words = L.nib_bytes / 4;
    nibble_kernel<<<(uint32_t)(sms ? sms * 4 : 1), 256, 0, s>>>(d_fp8, n, reinterpret_cast<uint32_t*>(blob + L.nib_off),
                                                                words);
    if (cudaGetLastError() != cudaSuccess) return ECF8_ERR_CUDA;
  }
  *blob_bytes = L.total;
  return ECF8_OK;
}

}  // extern "C"
