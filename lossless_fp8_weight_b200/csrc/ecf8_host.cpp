// Host side of the ECF8 library: exponent statistics, code construction,
// the blob encoder and the blob parser.  Encoding is offline work (the ECF8
// walkthrough's freeze_codebook, §5.1: built once after training, reused at
// inference), so it runs on CPU threads; the hot path is the GPU decoder in
// ecf8_decode.cu.
#include <omp.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <functional>
#include <queue>
#include <utility>
#include <vector>

#include "ecf8.h"
#include "ecf8_format.h"

using namespace ecf8;

namespace {

inline uint32_t load_le32(const uint8_t* p) {
  uint32_t v;
  memcpy(&v, p, 4);
  return v;
}
inline uint64_t load_le64(const uint8_t* p) {
  uint64_t v;
  memcpy(&v, p, 8);
  return v;
}
inline void store_le32(uint8_t* p, uint32_t v) { memcpy(p, &v, 4); }
inline void store_le64(uint8_t* p, uint64_t v) { memcpy(p, &v, 8); }

inline uint32_t exponent_of(uint8_t b) { return (b >> 3) & 15u; }

// Signs and mantissas of 8 weights in one word, laid out for the decoder:
// byte k holds weight k's sign (bit 7) and mantissa (bits 0-2), weight 4+k's
// mantissa (bits 4-6), and weight 4+((k+3)%4)'s sign (bit 3).  A decoder then
// takes weights 0-3 as word & 0x87878787 and weights 4-7 as the word rotated
// right by 4 bits & 0x87878787, each byte ready to OR with its exponent << 3.
inline uint32_t nibble_word(const uint8_t* b) {
  uint32_t v = 0;
  for (int k = 0; k < 4; ++k) {
    v |= (uint32_t)(b[k] & 0x87u) << (8 * k);
    v |= (uint32_t)(b[4 + k] & 7u) << (8 * k + 4);
    v |= (uint32_t)(b[4 + k] >> 7) << (8 * ((k + 1) & 3) + 3);
  }
  return v;
}

// Start of thread range p of `parts` over n weights.  Ranges start on whole
// 8-weight blocks, so the codes of a range (stream positions [i0, i1)) are the
// codes of its own weights [i0, i1), only reordered inside blocks.
size_t range_start(size_t n, int p, int parts) { return p >= parts ? n : (n * (size_t)p / parts) & ~(size_t)7; }

// Per-range exponent histograms, one per thread range, so that the encoder can
// also derive each range's bit length without a second pass.
void range_histograms(const uint8_t* x, size_t n, int parts, std::vector<uint64_t>& h) {
  h.assign((size_t)parts * 16, 0);
#pragma omp parallel for num_threads(parts) schedule(static, 1)
  for (int p = 0; p < parts; ++p) {
    const size_t i0 = range_start(n, p, parts), i1 = range_start(n, p + 1, parts);
    uint64_t c[4][16] = {};
    size_t i = i0;
    for (; i + 4 <= i1; i += 4) {
      ++c[0][exponent_of(x[i])];
      ++c[1][exponent_of(x[i + 1])];
      ++c[2][exponent_of(x[i + 2])];
      ++c[3][exponent_of(x[i + 3])];
    }
    for (; i < i1; ++i) ++c[0][exponent_of(x[i])];
    for (int s = 0; s < 16; ++s) h[(size_t)p * 16 + s] = c[0][s] + c[1][s] + c[2][s] + c[3][s];
  }
}

int thread_parts(size_t n) {
  const size_t min_per_thread = 1 << 20;
  int t = omp_get_max_threads();
  size_t want = (n + min_per_thread - 1) / min_per_thread;
  return (int)std::max<size_t>(1, std::min<size_t>((size_t)t, want));
}

// Huffman lengths; ties go to the smaller (weight, id), leaves have id =
// value and the k-th merged node id 16 + k.
void huffman(const uint64_t* hist, uint8_t* len) {
  using Item = std::pair<uint64_t, int>;
  std::priority_queue<Item, std::vector<Item>, std::greater<Item>> heap;
  int up[32];
  for (int i = 0; i < 32; ++i) up[i] = -1;
  for (int s = 0; s < 16; ++s) {
    len[s] = 0;
    if (hist[s]) heap.push({hist[s], s});
  }
  if (heap.size() == 1) {
    len[heap.top().second] = 1;
    return;
  }
  int next_id = 16;
  while (heap.size() > 1) {
    Item a = heap.top();
    heap.pop();
    Item b = heap.top();
    heap.pop();
    up[a.second] = next_id;
    up[b.second] = next_id;
    heap.push({a.first + b.first, next_id++});
  }
  for (int s = 0; s < 16; ++s) {
    if (!hist[s]) continue;
    int d = 0;
    for (int v = s; up[v] >= 0; v = up[v]) ++d;
    len[s] = (uint8_t)d;
  }
}

// Package-merge (Larmore and Hirschberg 1990) for a length limit: the coin
// collector's problem over denominations 2^-1 .. 2^-max_len.  Leaves are
// ordered by (weight, value); on equal weight a leaf precedes a package.
bool package_merge(const uint64_t* hist, int max_len, uint8_t* len) {
  struct Coin {
    uint64_t w;
    uint8_t uses[16];
  };
  std::vector<Coin> leaves;
  for (int s = 0; s < 16; ++s) {
    len[s] = 0;
    if (!hist[s]) continue;
    Coin c{hist[s], {}};
    c.uses[s] = 1;
    leaves.push_back(c);
  }
  const size_t k = leaves.size();
  if (k == 0) return true;
  if (k == 1) {
    for (int s = 0; s < 16; ++s)
      if (hist[s]) len[s] = 1;
    return true;
  }
  if (max_len < 1 || max_len > 16 || (size_t(1) << max_len) < k) return false;
  std::stable_sort(leaves.begin(), leaves.end(), [](const Coin& a, const Coin& b) { return a.w < b.w; });
  std::vector<Coin> row = leaves, merged;
  for (int depth = max_len; depth > 1; --depth) {
    std::vector<Coin> packs;
    for (size_t i = 0; i + 1 < row.size(); i += 2) {
      Coin p{row[i].w + row[i + 1].w, {}};
      for (int s = 0; s < 16; ++s) p.uses[s] = (uint8_t)(row[i].uses[s] + row[i + 1].uses[s]);
      packs.push_back(p);
    }
    merged.clear();
    std::merge(leaves.begin(), leaves.end(), packs.begin(), packs.end(), std::back_inserter(merged),
               [](const Coin& a, const Coin& b) { return a.w < b.w; });  // stable: leaves first on ties
    row.swap(merged);
  }
  for (size_t i = 0; i < 2 * k - 2; ++i)
    for (int s = 0; s < 16; ++s) len[s] = (uint8_t)(len[s] + row[i].uses[s]);
  return true;
}

// Canonical codes in (length, value) order; false if Kraft's sum exceeds 1.
bool canonical(const uint8_t* len, uint16_t* code) {
  uint32_t per_len[17] = {};
  uint64_t kraft = 0;
  for (int s = 0; s < 16; ++s) {
    if (len[s] > 16) return false;
    if (len[s]) {
      ++per_len[len[s]];
      kraft += 1ull << (16 - len[s]);
    }
  }
  if (kraft > (1ull << 16)) return false;
  uint32_t start[17] = {};
  uint32_t c = 0;
  for (int l = 1; l <= 16; ++l) {
    c = (c + per_len[l - 1]) << 1;
    start[l] = c;
  }
  for (int s = 0; s < 16; ++s) code[s] = len[s] ? (uint16_t)start[len[s]]++ : 0;
  return true;
}

// Writes codes [i0, i1) (stream order: code i is weight coded_weight(i, n))
// starting at stream bit bit0, and the gap and group offset of every chunk
// that starts in [bit0, bit1), where bit1 is the start of code i1 (the stream
// end for the last range).  Words shared with the neighbouring ranges are
// OR-ed atomically; the stream must start zeroed.
void pack_range(const uint8_t* x, size_t n, size_t i0, size_t i1, uint64_t bit0, uint64_t bit1, const uint8_t* len,
                const uint16_t* code, uint32_t C, uint32_t T, uint64_t chunks, uint32_t* stream, uint32_t* gaps,
                uint64_t* offs) {
  const uint64_t chunk_bits = 8ull * C;
  uint64_t chunk = (bit0 + chunk_bits - 1) / chunk_bits;  // first chunk starting at or after bit0
  uint64_t boundary = chunk * chunk_bits;
  auto put_gap = [&](uint64_t c, uint64_t gap, uint64_t first_code) {
    __atomic_fetch_or(&gaps[c / 8], (uint32_t)gap << (4 * (c % 8)), __ATOMIC_RELAXED);
    if (c % T == 0) offs[c / T] = first_code;
  };
  const uint64_t first_word = bit0 / 32;
  uint64_t word = first_word;
  uint64_t acc = 0;
  uint32_t nacc = (uint32_t)(bit0 % 32);  // leading bits owned by the previous range stay zero
  uint64_t pos = bit0;
  auto flush_word = [&](uint32_t v) {
    if (word == first_word)
      __atomic_fetch_or(&stream[stream_word_pos(word, C, T)], v, __ATOMIC_RELAXED);
    else
      stream[stream_word_pos(word, C, T)] = v;
    ++word;
  };
  for (size_t i = i0; i < i1; ++i) {
    const uint32_t e = exponent_of(x[coded_weight(i, n)]);
    if (boundary <= pos && chunk < chunks) {  // at most one boundary per code: codes <= 16 bits <= 8C
      put_gap(chunk, pos - boundary, i);
      ++chunk;
      boundary += chunk_bits;
    }
    const uint32_t l = len[e];
    acc = (acc << l) | code[e];
    nacc += l;
    pos += l;
    if (nacc >= 32) {
      nacc -= 32;
      flush_word((uint32_t)(acc >> nacc));
    }
  }
  if (nacc) {
    const uint32_t v = (uint32_t)(acc << (32 - nacc));
    __atomic_fetch_or(&stream[stream_word_pos(word, C, T)], v, __ATOMIC_RELAXED);  // shared with the next range
  }
  for (; boundary < bit1 && chunk < chunks; boundary += chunk_bits, ++chunk) put_gap(chunk, bit1 - boundary, i1);
}

// The 128-byte header of a blob; those bytes must already be zero.
void write_header(uint8_t* blob, const Layout& L, const ecf8_codebook* cb, uint8_t max_len, uint32_t chunk_bytes,
                  uint32_t group_chunks) {
  const uint64_t n = L.n;
  store_le32(blob + 0, kMagic);
  store_le32(blob + 4, kVersion);
  store_le64(blob + 8, n);
  store_le64(blob + 16, L.code_bits);
  store_le32(blob + 24, chunk_bytes);
  store_le32(blob + 28, group_chunks);
  store_le32(blob + 32, (uint32_t)L.groups);
  store_le32(blob + 36, 0);  // reserved
  store_le32(blob + 40, n ? max_len : 0);
  store_le32(blob + 44, kHeaderBytes);
  store_le64(blob + 48, 0);  // reserved
  store_le64(blob + 56, L.gaps_off);
  store_le64(blob + 64, L.groups_off);
  store_le64(blob + 72, L.stream_off);
  store_le64(blob + 80, L.nib_off);
  store_le64(blob + 88, L.total);
  memcpy(blob + 96, cb->len, 16);
}

bool codebook_ok(const ecf8_codebook* cb, uint16_t* code_out) {
  uint16_t code[16];
  if (!canonical(cb->len, code)) return false;
  for (int s = 0; s < 16; ++s)
    if (cb->len[s] && cb->code[s] != code[s]) return false;
  memcpy(code_out, code, sizeof(code));
  return true;
}

}  // namespace

extern "C" {

int ecf8_abi_version(void) { return ECF8_ABI_VERSION; }

const char* ecf8_strerror(int code) {
  switch (code) {
    case ECF8_OK: return "ok";
    case ECF8_ERR_ARG: return "invalid argument";
    case ECF8_ERR_FORMAT: return "malformed or inconsistent blob";
    case ECF8_ERR_CAPACITY: return "destination buffer too small";
    case ECF8_ERR_CODEBOOK: return "invalid codebook or exponent without a code";
    case ECF8_ERR_ALIGN: return "device pointer not 16-byte aligned";
    case ECF8_ERR_UNSUPPORTED: return "layout not implemented by the GPU kernels";
    case ECF8_ERR_CUDA: return "CUDA runtime error";
    case ECF8_ERR_WORKSPACE: return "workspace missing or too small";
    case ECF8_ERR_TOO_MANY: return "more tensors than the no-allocation decode table holds";
    case ECF8_ERR_CAPTURE: return "the call copies from host memory and its stream is capturing a graph";
    default: return "unknown error";
  }
}

int ecf8_histogram(const uint8_t* fp8, size_t n, uint64_t hist[16]) {
  if (!hist || (!fp8 && n)) return ECF8_ERR_ARG;
  const int parts = thread_parts(n);
  std::vector<uint64_t> h;
  range_histograms(fp8, n, parts, h);
  for (int s = 0; s < 16; ++s) {
    hist[s] = 0;
    for (int p = 0; p < parts; ++p) hist[s] += h[(size_t)p * 16 + s];
  }
  return ECF8_OK;
}

int ecf8_build_codebook(const uint64_t hist[16], uint32_t max_len, ecf8_codebook* out) {
  if (!hist || !out || max_len < 1 || max_len > 16) return ECF8_ERR_ARG;
  ecf8_codebook cb;
  memset(&cb, 0, sizeof(cb));
  huffman(hist, cb.len);
  uint32_t deepest = 0;
  for (int s = 0; s < 16; ++s) deepest = std::max<uint32_t>(deepest, cb.len[s]);
  if (deepest > max_len && !package_merge(hist, (int)max_len, cb.len)) return ECF8_ERR_CODEBOOK;
  if (!canonical(cb.len, cb.code)) return ECF8_ERR_CODEBOOK;
  for (int s = 0; s < 16; ++s) {
    cb.max_len = std::max<uint32_t>(cb.max_len, cb.len[s]);
    cb.n_symbols += cb.len[s] ? 1 : 0;
  }
  *out = cb;
  return ECF8_OK;
}

int ecf8_encoded_size(const uint64_t hist[16], size_t n, const ecf8_codebook* cb, uint32_t chunk_bytes,
                      uint32_t group_chunks, size_t* out_bytes) {
  if (!hist || !cb || !out_bytes) return ECF8_ERR_ARG;
  uint64_t bits = 0, total = 0;
  for (int s = 0; s < 16; ++s) {
    if (hist[s] && !cb->len[s]) return ECF8_ERR_CODEBOOK;
    bits += hist[s] * cb->len[s];
    total += hist[s];
  }
  if (total != n) return ECF8_ERR_ARG;
  Layout L;
  if (!compute_layout(n, bits, chunk_bytes, group_chunks, &L)) return ECF8_ERR_ARG;
  *out_bytes = L.total;
  return ECF8_OK;
}

size_t ecf8_encoded_size_bound(size_t n, uint32_t chunk_bytes, uint32_t group_chunks) {
  // every code is at most 16 bits long, so a stream never exceeds 16 n bits
  if (n > (SIZE_MAX >> 5)) return 0;
  Layout L;
  if (!compute_layout(n, 16ull * n, chunk_bytes, group_chunks, &L)) return 0;
  return (size_t)L.total;
}

int ecf8_encode(const uint8_t* fp8, size_t n, const ecf8_codebook* cb, uint32_t chunk_bytes, uint32_t group_chunks,
                void* blob_v, size_t cap, size_t* blob_bytes) {
  if (!cb || !blob_v || !blob_bytes || (!fp8 && n)) return ECF8_ERR_ARG;
  uint16_t code[16];
  if (!codebook_ok(cb, code)) return ECF8_ERR_CODEBOOK;
  const int parts = thread_parts(n);
  std::vector<uint64_t> h;
  range_histograms(fp8, n, parts, h);
  std::vector<uint64_t> range_bit(parts + 1, 0);
  for (int p = 0; p < parts; ++p) {
    uint64_t bits = 0;
    for (int s = 0; s < 16; ++s) {
      if (h[(size_t)p * 16 + s] && !cb->len[s]) return ECF8_ERR_CODEBOOK;
      bits += h[(size_t)p * 16 + s] * cb->len[s];
    }
    range_bit[p + 1] = range_bit[p] + bits;
  }
  Layout L;
  if (!compute_layout(n, range_bit[parts], chunk_bytes, group_chunks, &L)) return ECF8_ERR_ARG;
  if (cap < L.total) return ECF8_ERR_CAPACITY;
  uint8_t* blob = static_cast<uint8_t*>(blob_v);
  uint8_t max_len = 0;
  for (int s = 0; s < 16; ++s) max_len = std::max(max_len, cb->len[s]);

  // zero everything but the nibble section, which is written whole below
  memset(blob, 0, L.nib_off);
  write_header(blob, L, cb, max_len, chunk_bytes, group_chunks);

  uint32_t* stream = reinterpret_cast<uint32_t*>(blob + L.stream_off);
  uint32_t* gaps = reinterpret_cast<uint32_t*>(blob + L.gaps_off);
  uint64_t* offs = reinterpret_cast<uint64_t*>(blob + L.groups_off);
  const uint64_t chunks = L.groups * group_chunks;
#pragma omp parallel for num_threads(parts) schedule(static, 1)
  for (int p = 0; p < parts; ++p) {
    const size_t i0 = range_start(n, p, parts), i1 = range_start(n, p + 1, parts);
    pack_range(fp8, n, i0, i1, range_bit[p], range_bit[p + 1], cb->len, code, chunk_bytes, group_chunks, chunks,
               stream, gaps, offs);
  }
  // a chunk that starts exactly at the stream end, and every later one: gap 0,
  // and their groups begin at n
  const uint64_t chunk_bits = 8ull * chunk_bytes;
  for (uint64_t c = (L.code_bits + chunk_bits - 1) / chunk_bits; c < chunks; ++c)
    if (c % group_chunks == 0) offs[c / group_chunks] = n;
  offs[L.groups] = n;

  // sign/mantissa: 8 weights per little-endian u32 (see nibble_word)
  uint32_t* nib = reinterpret_cast<uint32_t*>(blob + L.nib_off);
  const long long words = (long long)(L.nib_bytes / 4);
#pragma omp parallel for num_threads(parts) schedule(static)
  for (long long w = 0; w < words; ++w) {
    const size_t i = (size_t)w * 8;
    uint8_t b[8] = {};
    for (int k = 0; k < 8 && i + k < n; ++k) b[k] = fp8[i + k];
    nib[w] = nibble_word(b);
  }
  *blob_bytes = L.total;
  return ECF8_OK;
}

int ecf8_blob_info(const void* blob_v, size_t size, ecf8_info* out) {
  if (!blob_v || !out) return ECF8_ERR_ARG;
  const uint8_t* b = static_cast<const uint8_t*>(blob_v);
  if (size < kHeaderBytes) return ECF8_ERR_FORMAT;
  if (load_le32(b) != kMagic || load_le32(b + 4) != kVersion || load_le32(b + 36) != 0 ||
      load_le32(b + 44) != kHeaderBytes)
    return ECF8_ERR_FORMAT;
  Layout L;
  const uint64_t n = load_le64(b + 8), code_bits = load_le64(b + 16);
  if (!compute_layout(n, code_bits, load_le32(b + 24), load_le32(b + 28), &L)) return ECF8_ERR_FORMAT;
  if (L.groups != load_le32(b + 32) || load_le64(b + 48) != 0 || L.gaps_off != load_le64(b + 56) ||
      L.groups_off != load_le64(b + 64) || L.stream_off != load_le64(b + 72) || L.nib_off != load_le64(b + 80) ||
      L.total != load_le64(b + 88) || L.total > size)
    return ECF8_ERR_FORMAT;
  ecf8_info info;
  memset(&info, 0, sizeof(info));
  memcpy(info.len, b + 96, 16);
  uint16_t code[16];
  if (!canonical(info.len, code)) return ECF8_ERR_CODEBOOK;
  uint32_t max_len = 0, present = 0;
  for (int s = 0; s < 16; ++s) {
    max_len = std::max<uint32_t>(max_len, info.len[s]);
    present += info.len[s] ? 1 : 0;
  }
  if (max_len != load_le32(b + 40)) return ECF8_ERR_FORMAT;
  if (n && (!present || code_bits < n || code_bits > 16 * n)) return ECF8_ERR_FORMAT;
  if (!n && code_bits) return ECF8_ERR_FORMAT;
  info.n = n;
  info.code_bits = code_bits;
  info.blob_bytes = L.total;
  info.gaps_off = L.gaps_off;
  info.groups_off = L.groups_off;
  info.stream_off = L.stream_off;
  info.nibbles_off = L.nib_off;
  info.chunk_bytes = L.C;
  info.group_chunks = L.T;
  info.n_groups = (uint32_t)L.groups;
  info.max_len = max_len;
  *out = info;
  return ECF8_OK;
}

}  // extern "C"

namespace ecf8 {

int prepare_blob(const ecf8_codebook* cb, const uint64_t hist[16], uint64_t n, uint32_t chunk_bytes,
                 uint32_t group_chunks, Layout* L, uint16_t code[16]) {
  if (!cb || !hist || !L || !code) return ECF8_ERR_ARG;
  if (!codebook_ok(cb, code)) return ECF8_ERR_CODEBOOK;
  uint64_t bits = 0, total = 0;
  for (int s = 0; s < 16; ++s) {
    if (hist[s] && !cb->len[s]) return ECF8_ERR_CODEBOOK;
    bits += hist[s] * cb->len[s];
    total += hist[s];
  }
  if (total != n) return ECF8_ERR_ARG;
  if (!compute_layout(n, bits, chunk_bytes, group_chunks, L)) return ECF8_ERR_ARG;
  return ECF8_OK;
}

void write_blob_prefix(uint8_t* blob, const Layout& L, const ecf8_codebook* cb, const uint16_t[16]) {
  memset(blob, 0, kHeaderBytes);
  uint8_t max_len = 0;
  for (int s = 0; s < 16; ++s) max_len = std::max(max_len, cb->len[s]);
  write_header(blob, L, cb, max_len, L.C, L.T);
}

}  // namespace ecf8
