/* BF16 variant CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, step-by-step definition of the DFloat11-style BF16 codec
 * (DFloat11 article §2: entropy-code the exponent field per tensor, keep the
 * sign and mantissa as they are; the same pipeline as the ECF8 walkthrough
 * §3.1.1-§3.2.1 with an 8-bit alphabet).  Only the tests, smoke() and
 * bench.py's CPU-baseline leg use it; the library never does.
 *
 * Readings where the pages are silent or garbled (the article's bit counts
 * for BF16 are inconsistent with the format; the plain reading of BF16 is 1
 * sign, 8 exponent and 7 mantissa bits):
 *  - symbol = exponent field (x >> 7) & 0xFF; kept byte = (x >> 15) << 7 | (x & 0x7F)
 *  - Huffman ties: merge the two nodes of least (weight, id); leaves have
 *    id = symbol, the k-th merged node id 256 + k.  One symbol gets length 1.
 *  - code lengths capped at 16 bits (the ECF8 walkthrough's cap): when the
 *    Huffman tree is deeper, package-merge (Larmore and Hirschberg 1990),
 *    leaves before packages on equal weight.
 *  - canonical code (RFC 1951 §3.2.2): codes in (length, symbol) order.
 *  - code stream, chunks, gaps and group offsets exactly as for ECF8:
 *    little-endian 32-bit words, MSB first; chunk c = bits [8Cc, 8C(c+1)),
 *    gap_c = first code start at or after 8Cc minus 8Cc (the stream end
 *    counts as a start; chunks wholly past it hold 0), 4 bits per chunk;
 *    group g = T chunks, off[g] = codes starting before bit 8CTg, off[G] = n.
 *  - blob: 128-byte header, then 256-byte-aligned sections: code lengths
 *    (256 bytes), gaps, group offsets, code stream (+16 pad bytes), the kept
 *    bytes (n, padded to 16).
 *
 * Parity pins live in tests/test_oracle_bf16_pins.py.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define NSYM 256
#define MAXLEN 16
#define HEADER 128
#define MAGIC 0x31314644u /* bytes 'D' 'F' '1' '1' */

static uint32_t rd32(const uint8_t* p) {
  return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}
static uint64_t rd64(const uint8_t* p) { return (uint64_t)rd32(p) | ((uint64_t)rd32(p + 4) << 32); }
static void wr32(uint8_t* p, uint32_t v) {
  p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); p[2] = (uint8_t)(v >> 16); p[3] = (uint8_t)(v >> 24);
}
static void wr64(uint8_t* p, uint64_t v) { wr32(p, (uint32_t)v); wr32(p + 4, (uint32_t)(v >> 32)); }
static uint64_t up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

/* ---------- split and join a BF16 value ---------- */
int bf16_exponent(uint16_t x) { return (x >> 7) & 0xFF; }
int bf16_kept(uint16_t x) { return ((x >> 15) << 7) | (x & 0x7F); }
uint16_t bf16_join(int e, int kept) { return (uint16_t)(((kept >> 7) << 15) | (e << 7) | (kept & 0x7F)); }

int bf16_histogram(const uint16_t* x, uint64_t n, uint64_t* hist) {
  for (int s = 0; s < NSYM; ++s) hist[s] = 0;
  for (uint64_t i = 0; i < n; ++i) hist[bf16_exponent(x[i])] += 1;
  return 0;
}

/* ---------- Huffman code lengths ---------- */
int bf16_huffman_lengths(const uint64_t* hist, uint8_t* len) {
  static uint64_t weight[2 * NSYM];
  static int parent[2 * NSYM], alive[2 * NSYM];
  int nodes = NSYM, live = 0;
  for (int s = 0; s < NSYM; ++s) {
    len[s] = 0;
    weight[s] = hist[s];
    parent[s] = -1;
    alive[s] = hist[s] > 0;
    live += alive[s];
  }
  if (live == 0) return 0;
  if (live == 1) {
    for (int s = 0; s < NSYM; ++s) if (alive[s]) len[s] = 1;
    return 0;
  }
  while (live > 1) {
    int pick[2];
    for (int k = 0; k < 2; ++k) {
      int best = -1;
      for (int id = 0; id < nodes; ++id) {
        if (!alive[id]) continue;
        if (best < 0 || weight[id] < weight[best]) best = id; /* ids ascend: ties keep the lower id */
      }
      pick[k] = best;
      alive[best] = 0;
    }
    weight[nodes] = weight[pick[0]] + weight[pick[1]];
    parent[nodes] = -1;
    alive[nodes] = 1;
    parent[pick[0]] = nodes;
    parent[pick[1]] = nodes;
    nodes += 1;
    live -= 1;
  }
  for (int s = 0; s < NSYM; ++s) {
    if (hist[s] == 0) continue;
    int d = 0;
    for (int v = s; parent[v] >= 0; v = parent[v]) d += 1;
    len[s] = (uint8_t)(d > 255 ? 255 : d);
  }
  return 0;
}

/* ---------- package-merge under a length limit ---------- */
typedef struct { uint64_t w; uint16_t cnt[NSYM]; } pm_item;

int bf16_package_merge_lengths(const uint64_t* hist, int max_len, uint8_t* len) {
  static pm_item leaves[NSYM], list[2 * NSYM], next[2 * NSYM], pkg[NSYM];
  int k = 0;
  for (int s = 0; s < NSYM; ++s) len[s] = 0;
  for (int s = 0; s < NSYM; ++s) {
    if (hist[s] == 0) continue;
    memset(&leaves[k], 0, sizeof(pm_item));
    leaves[k].w = hist[s];
    leaves[k].cnt[s] = 1;
    k += 1;
  }
  if (k == 0) return 0;
  if (k == 1) { for (int s = 0; s < NSYM; ++s) if (hist[s]) len[s] = 1; return 0; }
  if (max_len < 1 || max_len > MAXLEN || (1 << max_len) < k) return -1;
  for (int i = 1; i < k; ++i) { /* insertion sort by (weight, symbol) */
    pm_item t = leaves[i];
    int j = i - 1;
    while (j >= 0 && leaves[j].w > t.w) { leaves[j + 1] = leaves[j]; --j; }
    leaves[j + 1] = t;
  }
  int nl = k;
  for (int i = 0; i < k; ++i) list[i] = leaves[i];
  for (int level = 1; level < max_len; ++level) {
    int np = nl / 2;
    for (int i = 0; i < np; ++i) {
      pkg[i].w = list[2 * i].w + list[2 * i + 1].w;
      for (int s = 0; s < NSYM; ++s) pkg[i].cnt[s] = (uint16_t)(list[2 * i].cnt[s] + list[2 * i + 1].cnt[s]);
    }
    int a = 0, b = 0, m = 0;
    while (a < k || b < np) { /* merge; a leaf goes first on equal weight */
      if (b >= np || (a < k && leaves[a].w <= pkg[b].w)) next[m++] = leaves[a++];
      else next[m++] = pkg[b++];
    }
    nl = m;
    for (int i = 0; i < nl; ++i) list[i] = next[i];
  }
  for (int i = 0; i < 2 * k - 2; ++i)
    for (int s = 0; s < NSYM; ++s) len[s] = (uint8_t)(len[s] + list[i].cnt[s]);
  return 0;
}

int bf16_code_lengths(const uint64_t* hist, int max_len, uint8_t* len) {
  if (bf16_huffman_lengths(hist, len) != 0) return -1;
  int deepest = 0;
  for (int s = 0; s < NSYM; ++s) if (len[s] > deepest) deepest = len[s];
  if (deepest <= max_len) return 0;
  return bf16_package_merge_lengths(hist, max_len, len);
}

int bf16_canonical_codes(const uint8_t* len, uint32_t* code) {
  int count[MAXLEN + 2] = {0};
  uint32_t next[MAXLEN + 2] = {0};
  for (int s = 0; s < NSYM; ++s) {
    if (len[s] > MAXLEN) return -1;
    if (len[s]) count[len[s]] += 1;
  }
  uint32_t c = 0;
  for (int l = 1; l <= MAXLEN; ++l) {
    c = (c + (uint32_t)count[l - 1]) << 1;
    next[l] = c;
  }
  for (int s = 0; s < NSYM; ++s) code[s] = len[s] ? next[len[s]]++ : 0;
  return 0;
}

/* ---------- layout ---------- */
typedef struct {
  uint64_t n, code_bits, groups, lens_off, gaps_off, gaps_size, groups_off, stream_off, stream_size, kept_off, kept_size, total;
} layout_t;

static int make_layout(uint64_t n, uint64_t code_bits, uint32_t C, uint32_t T, layout_t* L) {
  if (C < 4 || C % 4 || T < 1) return -1;
  L->n = n;
  L->code_bits = code_bits;
  uint64_t gbits = 8ull * C * T;
  L->groups = (code_bits + gbits - 1) / gbits;
  uint64_t chunks = L->groups * T;
  L->lens_off = up(HEADER, 256);
  L->gaps_off = up(L->lens_off + NSYM, 256);
  L->gaps_size = up((chunks + 7) / 8 * 4, 16);
  L->groups_off = up(L->gaps_off + L->gaps_size, 256);
  L->stream_off = up(L->groups_off + 8 * (L->groups + 1), 256);
  L->stream_size = n ? chunks * C + 16 : 0;
  L->kept_off = up(L->stream_off + L->stream_size, 256);
  L->kept_size = up(n, 16);
  L->total = L->kept_off + L->kept_size;
  return 0;
}

static void set_bit(uint8_t* stream, uint64_t i) {
  uint8_t* p = stream + 4 * (i / 32);
  wr32(p, rd32(p) | (1u << (31 - (i % 32))));
}
static int get_bit(const uint8_t* stream, uint64_t i) {
  return (int)((rd32(stream + 4 * (i / 32)) >> (31 - (i % 32))) & 1u);
}

uint64_t bf16_encoded_size(const uint16_t* x, uint64_t n, const uint8_t* len, uint32_t C, uint32_t T) {
  uint64_t bits = 0;
  for (uint64_t i = 0; i < n; ++i) bits += len[bf16_exponent(x[i])];
  layout_t L;
  if (make_layout(n, bits, C, T, &L) != 0) return 0;
  return L.total;
}

/* Encode with the given code lengths: 0, or -1 (lengths), -2 (exponent
 * without a code), -3 (capacity), -4 (a gap above 15). */
int bf16_encode(const uint16_t* x, uint64_t n, const uint8_t* len, uint32_t C, uint32_t T, uint8_t* blob,
                uint64_t cap, uint64_t* size) {
  uint32_t code[NSYM];
  int max_len = 0;
  for (int s = 0; s < NSYM; ++s) if (len[s] > max_len) max_len = len[s];
  if (max_len > MAXLEN || bf16_canonical_codes(len, code) != 0) return -1;
  uint64_t bits = 0;
  for (uint64_t i = 0; i < n; ++i) {
    if (len[bf16_exponent(x[i])] == 0) return -2;
    bits += len[bf16_exponent(x[i])];
  }
  layout_t L;
  if (make_layout(n, bits, C, T, &L) != 0) return -1;
  if (cap < L.total) return -3;
  memset(blob, 0, L.total);
  wr32(blob + 0, MAGIC);
  wr32(blob + 4, 1);
  wr64(blob + 8, n);
  wr64(blob + 16, bits);
  wr32(blob + 24, C);
  wr32(blob + 28, T);
  wr32(blob + 32, (uint32_t)L.groups);
  wr32(blob + 36, (uint32_t)max_len);
  wr64(blob + 40, L.lens_off);
  wr64(blob + 48, L.gaps_off);
  wr64(blob + 56, L.groups_off);
  wr64(blob + 64, L.stream_off);
  wr64(blob + 72, L.kept_off);
  wr64(blob + 80, L.total);
  memcpy(blob + L.lens_off, len, NSYM);

  uint8_t* stream = blob + L.stream_off;
  uint8_t* gaps = blob + L.gaps_off;
  uint8_t* offs = blob + L.groups_off;
  uint64_t chunk_bits = 8ull * C, chunks = L.groups * T, next_chunk = 0, pos = 0;
  for (uint64_t i = 0; i <= n; ++i) {
    while (next_chunk < chunks && next_chunk * chunk_bits <= pos) {
      uint64_t gap = pos - next_chunk * chunk_bits;
      if (gap > 15) return -4;
      uint8_t* gp = gaps + 4 * (next_chunk / 8);
      wr32(gp, rd32(gp) | ((uint32_t)gap << (4 * (next_chunk % 8))));
      if (next_chunk % T == 0) wr64(offs + 8 * (next_chunk / T), i);
      next_chunk += 1;
    }
    if (i == n) break;
    int e = bf16_exponent(x[i]);
    for (int b = len[e] - 1; b >= 0; --b) {
      if ((code[e] >> b) & 1u) set_bit(stream, pos);
      pos += 1;
    }
  }
  for (; next_chunk < chunks; ++next_chunk)
    if (next_chunk % T == 0) wr64(offs + 8 * (next_chunk / T), n);
  wr64(offs + 8 * L.groups, n);
  for (uint64_t i = 0; i < n; ++i) blob[L.kept_off + i] = (uint8_t)bf16_kept(x[i]);
  *size = L.total;
  return 0;
}

/* Bit-serial decode of the whole stream, ignoring gaps and offsets: 0, or
 * -1 (header), -2 (bits that match no code), -3 (length mismatch). */
int bf16_decode(const uint8_t* blob, uint64_t size, uint16_t* out, uint64_t n) {
  if (size < HEADER || rd32(blob) != MAGIC || rd32(blob + 4) != 1) return -1;
  if (rd64(blob + 8) != n) return -3;
  uint64_t bits = rd64(blob + 16), stream_off = rd64(blob + 64), kept_off = rd64(blob + 72);
  const uint8_t* len = blob + rd64(blob + 40);
  uint32_t code[NSYM];
  if (bf16_canonical_codes(len, code) != 0) return -1;
  uint64_t pos = 0;
  for (uint64_t i = 0; i < n; ++i) {
    uint32_t c = 0;
    int sym = -1;
    for (int l = 1; l <= MAXLEN && pos + (uint64_t)l <= bits; ++l) {
      c = (c << 1) | (uint32_t)get_bit(blob + stream_off, pos + (uint64_t)(l - 1));
      for (int s = 0; s < NSYM; ++s)
        if (len[s] == l && code[s] == c) { sym = s; break; }
      if (sym >= 0) { pos += (uint64_t)l; break; }
    }
    if (sym < 0) return -2;
    out[i] = bf16_join(sym, blob[kept_off + i]);
  }
  return pos == bits ? 0 : -3;
}
