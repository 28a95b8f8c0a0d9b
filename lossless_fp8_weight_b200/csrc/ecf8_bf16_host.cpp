// Host side of the BF16 variant (DFloat11 article §2: the exponent field
// entropy coded per tensor, sign and mantissa kept): code lengths for the
// 256-symbol exponent alphabet (Huffman, package-merge under the 16-bit cap),
// canonical codes, the blob (the same bytes as the oracle's), the blob parser,
// and the decode table the GPU kernel walks: one entry per (tree node,
// 4-bit nibble) giving the exponents whose codes end in the nibble and the
// node after it.
#include <omp.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "ecf8.h"

namespace {

constexpr uint32_t kMagic = 0x31314644u;  // "DF11"
constexpr uint32_t kHeader = 128;
constexpr int kSym = 256, kMaxLen = 16;

uint32_t ld32(const uint8_t* p) { uint32_t v; memcpy(&v, p, 4); return v; }
uint64_t ld64(const uint8_t* p) { uint64_t v; memcpy(&v, p, 8); return v; }
void st32(uint8_t* p, uint32_t v) { memcpy(p, &v, 4); }
void st64(uint8_t* p, uint64_t v) { memcpy(p, &v, 8); }
uint64_t up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

struct Layout {
  uint64_t groups, lens_off, gaps_off, gaps_size, groups_off, stream_off, stream_size, kept_off, total;
};

bool layout(uint64_t n, uint64_t bits, uint32_t C, uint32_t T, Layout* L) {
  if (C < 4 || C % 4 || T < 1) return false;
  const uint64_t gbits = 8ull * C * T;
  L->groups = (bits + gbits - 1) / gbits;
  if (L->groups > 0xFFFFFFFFull) return false;
  const uint64_t chunks = L->groups * T;
  L->lens_off = up(kHeader, 256);
  L->gaps_off = up(L->lens_off + kSym, 256);
  L->gaps_size = up((chunks + 7) / 8 * 4, 16);
  L->groups_off = up(L->gaps_off + L->gaps_size, 256);
  L->stream_off = up(L->groups_off + 8 * (L->groups + 1), 256);
  L->stream_size = n ? chunks * C + 16 : 0;
  L->kept_off = up(L->stream_off + L->stream_size, 256);
  L->total = L->kept_off + up(n, 16);
  return true;
}

// Huffman lengths: repeatedly merge the two least (weight, id) nodes.
void huffman(const uint64_t* h, uint8_t* len) {
  struct Node { uint64_t w; int id; };
  std::vector<Node> live;
  std::vector<int> parent(2 * kSym, -1);
  for (int s = 0; s < kSym; ++s) {
    len[s] = 0;
    if (h[s]) live.push_back({h[s], s});
  }
  if (live.empty()) return;
  if (live.size() == 1) { len[live[0].id] = 1; return; }
  int next = kSym;
  auto less = [](const Node& a, const Node& b) { return a.w != b.w ? a.w < b.w : a.id < b.id; };
  while (live.size() > 1) {
    std::sort(live.begin(), live.end(), less);
    const Node a = live[0], b = live[1];
    live.erase(live.begin(), live.begin() + 2);
    parent[a.id] = next;
    parent[b.id] = next;
    live.push_back({a.w + b.w, next++});
  }
  for (int s = 0; s < kSym; ++s) {
    if (!h[s]) continue;
    int d = 0;
    for (int v = s; parent[v] >= 0; v = parent[v]) ++d;
    len[s] = (uint8_t)std::min(d, 255);
  }
}

// Package-merge (Larmore-Hirschberg): leaves before packages on equal weight.
bool package_merge(const uint64_t* h, int limit, uint8_t* len) {
  struct Item { uint64_t w; std::vector<uint16_t> cnt; };
  std::vector<Item> leaves;
  for (int s = 0; s < kSym; ++s) {
    len[s] = 0;
    if (h[s]) {
      Item it{h[s], std::vector<uint16_t>(kSym, 0)};
      it.cnt[s] = 1;
      leaves.push_back(std::move(it));
    }
  }
  const int k = (int)leaves.size();
  if (k == 0) return true;
  if (k == 1) {
    for (int s = 0; s < kSym; ++s) if (h[s]) len[s] = 1;
    return true;
  }
  if (limit < 1 || limit > kMaxLen || (1 << limit) < k) return false;
  std::stable_sort(leaves.begin(), leaves.end(), [](const Item& a, const Item& b) { return a.w < b.w; });
  std::vector<Item> list = leaves;
  for (int level = 1; level < limit; ++level) {
    std::vector<Item> pkg;
    for (size_t i = 0; i + 1 < list.size(); i += 2) {
      Item p{list[i].w + list[i + 1].w, std::vector<uint16_t>(kSym)};
      for (int s = 0; s < kSym; ++s) p.cnt[s] = (uint16_t)(list[i].cnt[s] + list[i + 1].cnt[s]);
      pkg.push_back(std::move(p));
    }
    std::vector<Item> merged;
    size_t a = 0, b = 0;
    while (a < leaves.size() || b < pkg.size()) {
      if (b >= pkg.size() || (a < leaves.size() && leaves[a].w <= pkg[b].w)) merged.push_back(leaves[a++]);
      else merged.push_back(pkg[b++]);
    }
    list.swap(merged);
  }
  for (int i = 0; i < 2 * k - 2; ++i)
    for (int s = 0; s < kSym; ++s) len[s] = (uint8_t)(len[s] + list[i].cnt[s]);
  return true;
}

// The lengths the blob parser accepts: at most 16 bits, and a complete
// prefix code (Kraft sum 1) unless a single value is present.
bool valid_lengths(const uint8_t* len) {
  uint64_t kraft = 0;
  int present = 0;
  for (int s = 0; s < kSym; ++s) {
    if (len[s] > kMaxLen) return false;
    if (len[s]) {
      kraft += 1ull << (kMaxLen - len[s]);
      ++present;
    }
  }
  return present == 0 || (present == 1 ? kraft <= (1ull << kMaxLen) : kraft == (1ull << kMaxLen));
}

bool canonical(const uint8_t* len, uint32_t* code) {
  int count[kMaxLen + 2] = {0};
  uint32_t next[kMaxLen + 2] = {0};
  for (int s = 0; s < kSym; ++s) {
    if (len[s] > kMaxLen) return false;
    if (len[s]) ++count[len[s]];
  }
  uint32_t c = 0;
  for (int l = 1; l <= kMaxLen; ++l) {
    c = (c + (uint32_t)count[l - 1]) << 1;
    next[l] = c;
  }
  for (int s = 0; s < kSym; ++s) code[s] = len[s] ? next[len[s]]++ : 0;
  return true;
}

// Host threads for n weights: ranges of at least 1M weights.
int parts_for(size_t n) {
  const size_t per = (size_t)1 << 20;
  const size_t want = (n + per - 1) / per;
  const size_t t = (size_t)std::max(1, omp_get_max_threads());
  return (int)std::max<size_t>(1, std::min(t, want));
}

// Code bits of weights [i0, i1); false when an exponent there has no code.
bool range_bits(const uint16_t* x, size_t i0, size_t i1, const uint8_t* len, uint64_t* bits) {
  uint64_t b = 0;
  bool ok = true;
  for (size_t i = i0; i < i1; ++i) {
    const uint8_t l = len[(x[i] >> 7) & 0xFF];
    ok &= l != 0;
    b += l;
  }
  *bits = b;
  return ok;
}

// Bits of each of `parts` equal weight ranges, as a prefix sum (range_bit[p]
// is where range p's first code starts); false when an exponent has no code.
bool prefix_bits(const uint16_t* x, size_t n, const uint8_t* len, int parts, std::vector<uint64_t>* range_bit) {
  range_bit->assign(parts + 1, 0);
  std::vector<uint64_t> bits(parts, 0);
  std::vector<char> ok(parts, 1);
#pragma omp parallel for num_threads(parts) schedule(static, 1)
  for (int p = 0; p < parts; ++p)
    ok[p] = range_bits(x, n * (size_t)p / parts, n * (size_t)(p + 1) / parts, len, &bits[p]) ? 1 : 0;
  for (int p = 0; p < parts; ++p) {
    if (!ok[p]) return false;
    (*range_bit)[p + 1] = (*range_bit)[p] + bits[p];
  }
  return true;
}

// Codes of weights [i0, i1) into the stream from bit bit0, with the gap and
// group offset of every chunk that starts in [bit0, bit1) (bit1: where code
// i1 starts, or the stream end).  Words shared with the neighbouring ranges
// are OR-ed atomically into a zeroed stream.
void pack(const uint16_t* x, size_t i0, size_t i1, uint64_t bit0, uint64_t bit1, const uint8_t* len,
          const uint32_t* code, uint64_t chunk_bits, uint32_t T, uint64_t chunks, uint32_t* stream, uint32_t* gaps,
          uint64_t* offs) {
  uint64_t chunk = (bit0 + chunk_bits - 1) / chunk_bits;  // the first chunk starting at or after bit0
  uint64_t boundary = chunk * chunk_bits;
  auto put_gap = [&](uint64_t c, uint64_t gap, uint64_t first_code) {
    __atomic_fetch_or(&gaps[c / 8], (uint32_t)gap << (4 * (c % 8)), __ATOMIC_RELAXED);
    if (c % T == 0) offs[c / T] = first_code;
  };
  const uint64_t first_word = bit0 / 32;
  uint64_t word = first_word, pos = bit0, acc = 0;
  uint32_t nacc = (uint32_t)(bit0 % 32);  // the previous range's bits of the first word stay zero here
  for (size_t i = i0; i < i1; ++i) {
    while (chunk < chunks && boundary <= pos) {  // at most once: a code is <= 16 bits, a chunk >= 32
      put_gap(chunk, pos - boundary, i);
      ++chunk;
      boundary += chunk_bits;
    }
    const uint32_t e = (x[i] >> 7) & 0xFF;
    acc = (acc << len[e]) | code[e];
    nacc += len[e];
    pos += len[e];
    if (nacc >= 32) {
      nacc -= 32;
      const uint32_t v = (uint32_t)(acc >> nacc);
      if (word == first_word)
        __atomic_fetch_or(&stream[word], v, __ATOMIC_RELAXED);
      else
        stream[word] = v;
      ++word;
    }
  }
  if (nacc) __atomic_fetch_or(&stream[word], (uint32_t)(acc << (32 - nacc)), __ATOMIC_RELAXED);
  for (; chunk < chunks && boundary < bit1; ++chunk, boundary += chunk_bits) put_gap(chunk, bit1 - boundary, i1);
}

}  // namespace

extern "C" {

int ecf8_bf16_code_lengths(const uint16_t* x, size_t n, uint32_t max_len, uint8_t len[256]) {
  if (!len || (!x && n) || max_len < 1 || max_len > kMaxLen) return ECF8_ERR_ARG;
  const int parts = parts_for(n);
  std::vector<uint64_t> ph((size_t)parts * kSym, 0), h(kSym, 0);
#pragma omp parallel for num_threads(parts) schedule(static, 1)
  for (int p = 0; p < parts; ++p) {
    uint64_t* hp = ph.data() + (size_t)p * kSym;
    for (size_t i = n * (size_t)p / parts, e = n * (size_t)(p + 1) / parts; i < e; ++i) ++hp[(x[i] >> 7) & 0xFF];
  }
  for (int p = 0; p < parts; ++p)
    for (int v = 0; v < kSym; ++v) h[v] += ph[(size_t)p * kSym + v];
  huffman(h.data(), len);
  int deepest = 0;
  for (int s = 0; s < kSym; ++s) deepest = std::max<int>(deepest, len[s]);
  if (deepest > (int)max_len && !package_merge(h.data(), (int)max_len, len)) return ECF8_ERR_CODEBOOK;
  return ECF8_OK;
}

int ecf8_bf16_encoded_size(const uint16_t* x, size_t n, const uint8_t len[256], uint32_t chunk_bytes,
                           uint32_t group_chunks, size_t* bytes) {
  if (!len || !bytes || (!x && n)) return ECF8_ERR_ARG;
  if (!valid_lengths(len)) return ECF8_ERR_CODEBOOK;
  std::vector<uint64_t> range_bit;
  if (!prefix_bits(x, n, len, parts_for(n), &range_bit)) return ECF8_ERR_CODEBOOK;
  Layout L;
  if (!layout(n, range_bit.back(), chunk_bytes, group_chunks, &L)) return ECF8_ERR_ARG;
  *bytes = L.total;
  return ECF8_OK;
}

int ecf8_bf16_encode(const uint16_t* x, size_t n, const uint8_t len[256], uint32_t chunk_bytes,
                     uint32_t group_chunks, void* blob_v, size_t cap, size_t* bytes) {
  if (!len || !blob_v || !bytes || (!x && n)) return ECF8_ERR_ARG;
  uint32_t code[kSym];
  if (!valid_lengths(len) || !canonical(len, code)) return ECF8_ERR_CODEBOOK;
  int max_len = 0;
  for (int s = 0; s < kSym; ++s) max_len = std::max<int>(max_len, len[s]);
  const int parts = parts_for(n);
  std::vector<uint64_t> range_bit;
  if (!prefix_bits(x, n, len, parts, &range_bit)) return ECF8_ERR_CODEBOOK;
  const uint64_t bits = range_bit.back();
  Layout L;
  if (!layout(n, bits, chunk_bytes, group_chunks, &L)) return ECF8_ERR_ARG;
  if (cap < L.total) return ECF8_ERR_CAPACITY;
  uint8_t* b = static_cast<uint8_t*>(blob_v);
  memset(b, 0, L.total);
  st32(b + 0, kMagic);
  st32(b + 4, 1);
  st64(b + 8, n);
  st64(b + 16, bits);
  st32(b + 24, chunk_bytes);
  st32(b + 28, group_chunks);
  st32(b + 32, (uint32_t)L.groups);
  st32(b + 36, (uint32_t)max_len);
  st64(b + 40, L.lens_off);
  st64(b + 48, L.gaps_off);
  st64(b + 56, L.groups_off);
  st64(b + 64, L.stream_off);
  st64(b + 72, L.kept_off);
  st64(b + 80, L.total);
  memcpy(b + L.lens_off, len, kSym);
  uint32_t* stream = reinterpret_cast<uint32_t*>(b + L.stream_off);
  uint32_t* gaps = reinterpret_cast<uint32_t*>(b + L.gaps_off);
  uint64_t* offs = reinterpret_cast<uint64_t*>(b + L.groups_off);
  const uint64_t chunk_bits = 8ull * chunk_bytes, chunks = L.groups * group_chunks;
#pragma omp parallel for num_threads(parts) schedule(static, 1)
  for (int p = 0; p < parts; ++p)
    pack(x, n * (size_t)p / parts, n * (size_t)(p + 1) / parts, range_bit[p], range_bit[p + 1], len, code,
         chunk_bits, group_chunks, chunks, stream, gaps, offs);
  // a chunk that starts at or after the stream end: gap 0, its group begins at n
  for (uint64_t c = (bits + chunk_bits - 1) / chunk_bits; c < chunks; ++c)
    if (c % group_chunks == 0) offs[c / group_chunks] = n;
  offs[L.groups] = n;
  uint8_t* kept = b + L.kept_off;
  const long long nn = (long long)n;
#pragma omp parallel for num_threads(parts) schedule(static)
  for (long long i = 0; i < nn; ++i) kept[i] = (uint8_t)(((x[i] >> 15) << 7) | (x[i] & 0x7F));
  *bytes = L.total;
  return ECF8_OK;
}

int ecf8_bf16_blob_info(const void* blob_v, size_t size, ecf8_bf16_info* out) {
  if (!blob_v || !out) return ECF8_ERR_ARG;
  const uint8_t* b = static_cast<const uint8_t*>(blob_v);
  if (size < kHeader || ld32(b) != kMagic || ld32(b + 4) != 1) return ECF8_ERR_FORMAT;
  ecf8_bf16_info I;
  memset(&I, 0, sizeof(I));
  I.n = ld64(b + 8);
  I.code_bits = ld64(b + 16);
  I.chunk_bytes = ld32(b + 24);
  I.group_chunks = ld32(b + 28);
  I.n_groups = ld32(b + 32);
  I.max_len = ld32(b + 36);
  Layout L;
  if (!layout(I.n, I.code_bits, I.chunk_bytes, I.group_chunks, &L)) return ECF8_ERR_FORMAT;
  if (L.groups != I.n_groups || L.lens_off != ld64(b + 40) || L.gaps_off != ld64(b + 48) ||
      L.groups_off != ld64(b + 56) || L.stream_off != ld64(b + 64) || L.kept_off != ld64(b + 72) ||
      L.total != ld64(b + 80) || L.total > size)
    return ECF8_ERR_FORMAT;
  memcpy(I.len, b + L.lens_off, kSym);
  uint64_t kraft = 0;
  int present = 0, deepest = 0;
  for (int s = 0; s < kSym; ++s) {
    if (I.len[s] > kMaxLen) return ECF8_ERR_CODEBOOK;
    if (I.len[s]) {
      kraft += 1ull << (kMaxLen - I.len[s]);
      ++present;
      deepest = std::max<int>(deepest, I.len[s]);
    }
  }
  if (I.n && (present == 0 || kraft > (1ull << kMaxLen) || (present > 1 && kraft != (1ull << kMaxLen))))
    return ECF8_ERR_CODEBOOK;
  if ((uint32_t)deepest != I.max_len) return ECF8_ERR_FORMAT;
  I.blob_bytes = L.total;
  I.lens_off = L.lens_off;
  I.gaps_off = L.gaps_off;
  I.groups_off = L.groups_off;
  I.stream_off = L.stream_off;
  I.kept_off = L.kept_off;
  *out = I;
  return ECF8_OK;
}

size_t ecf8_bf16_table_bytes(void) { return 256 * 16 * 8; }

}  // extern "C"

namespace {

// The code tree as the table builder numbers it: node 0 is the root; the
// internal nodes at depth l are the code values first[l] + count[l] + k
// (k < nint[l]) numbered from ibase[l]; with a single exponent present, node
// d means d zero bits read.  nodes = the number of nodes, also the index of
// the error node.
struct Tree {
  uint32_t count[kMaxLen + 1] = {0}, first[kMaxLen + 1] = {0}, base[kMaxLen + 1] = {0};
  uint32_t nint[kMaxLen + 1] = {0}, ibase[kMaxLen + 1] = {0};
  int max_len = 0, present = 0;
  std::vector<int> sorted;
  uint32_t nodes = 0;
  bool ok = false;
};

// with_order: also list the values in canonical order (the table builder
// needs it; the node count does not)
Tree make_tree(const uint8_t* len, bool with_order) {
  Tree t;
  for (int s = 0; s < kSym; ++s)
    if (len[s] && len[s] <= kMaxLen) { ++t.count[len[s]]; ++t.present; t.max_len = std::max<int>(t.max_len, len[s]); }
  if (with_order)
    for (int l = 1; l <= kMaxLen; ++l)
      for (int s = 0; s < kSym; ++s)
        if (len[s] == l) t.sorted.push_back(s);
  uint32_t c = 0, b = 0;
  for (int l = 1; l <= kMaxLen; ++l) {
    c = (c + t.count[l - 1]) << 1;
    t.first[l] = c;
    t.base[l] = b;
    b += t.count[l];
  }
  t.nint[0] = 1;
  uint32_t states = 1;
  t.ok = t.present >= 1;
  for (int l = 1; l <= kMaxLen; ++l) {
    long long k = l < t.max_len ? 2ll * t.nint[l - 1] - t.count[l] : 0;
    if (k < 0) { t.ok = false; k = 0; }
    t.nint[l] = (uint32_t)k;
    t.ibase[l] = states;
    states += (uint32_t)k;
  }
  if (t.present == 1) states = (uint32_t)t.max_len;
  if (states > 255) t.ok = false;
  t.nodes = t.ok ? states : 0;
  return t;
}

}  // namespace

extern "C" {

uint32_t ecf8_bf16_table_nodes(const ecf8_bf16_info* info) { return info ? make_tree(info->len, false).nodes : 0; }

// Entry (node s, nibble v) at index s * 16 + v: x = the exponents whose codes
// end inside the nibble, 8 bits each, first lowest; y = (next node << 7) |
// (8 * count) << 16, i.e. the next node's byte offset in the table and the
// bits the exponents take when packed a byte each.  Every entry of the
// error node (index = nodes) and of the unused nodes above it leads to the
// error node.
int ecf8_bf16_build_table(const ecf8_bf16_info* info, void* h_table) {
  if (!info || !h_table) return ECF8_ERR_ARG;
  const Tree T = make_tree(info->len, true);
  const uint32_t err = T.nodes;
  auto step = [&](uint32_t s, uint32_t bit, int* sym) -> uint32_t {
    *sym = -1;
    if (!T.ok || s >= T.nodes) return err;
    if (T.present == 1) {  // one exponent, code max_len zero bits: a 1 bit is no code
      if (bit) return err;
      if ((int)s + 1 < T.max_len) return s + 1;
      *sym = T.sorted[0];
      return 0;
    }
    uint32_t l = 0, v = 0;
    for (int d = 1; d < T.max_len; ++d)
      if (s >= T.ibase[d] && s < T.ibase[d] + T.nint[d]) { l = (uint32_t)d; v = T.first[d] + T.count[d] + (s - T.ibase[d]); }
    v = 2 * v + bit;
    ++l;
    const uint32_t r = v - T.first[l];
    if (r < T.count[l]) { *sym = T.sorted[T.base[l] + r]; return 0; }
    if ((int)l >= T.max_len) return err;
    return T.ibase[l] + (v - T.first[l] - T.count[l]);
  };
  uint32_t* t = static_cast<uint32_t*>(h_table);
  for (uint32_t s = 0; s < 256; ++s)
    for (uint32_t nib = 0; nib < 16; ++nib) {
      uint32_t node = s, syms = 0, k = 0;
      for (int i = 3; i >= 0 && node != err; --i) {
        int sym;
        node = step(node, (nib >> i) & 1u, &sym);
        if (sym >= 0) syms |= (uint32_t)sym << (8 * k++);
      }
      const bool bad = node == err;
      t[2 * (s * 16 + nib)] = bad ? 0 : syms;
      t[2 * (s * 16 + nib) + 1] = bad ? (err << 7) : ((node << 7) | ((8 * k) << 16));
    }
  return ECF8_OK;
}

}  // extern "C"
