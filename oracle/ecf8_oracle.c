/*
 * ECF8 CPU ORACLE -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, bit-serial implementation of the ECF8 codec for FP8 E4M3
 * weights, used to prove the GPU decoder right.  Only the tests, the smoke
 * check and the benchmark's CPU-baseline leg may load it.  It shares no code
 * with the library under lossless_fp8_weight_b200/: the blob layout below is
 * written out here on its own, from the format description.
 *
 * Method (ECF8 walkthrough, "ECF8 浮点数压缩技术" p1 §3.1.1; arXiv 2510.02676
 * abstract): the 4-bit exponent field of each E4M3 weight is entropy coded
 * with a per-tensor Huffman code of at most 16 bits; sign and mantissa are
 * stored raw.  Decoding must give back every byte exactly (p1 §1, abstract:
 * "bit-exact", "no deviation in model outputs").
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - symbol = raw biased exponent field (b >> 3) & 15; nibble = (b >> 7) << 3 | (b & 7)
 *  - Huffman ties: merge the two nodes of least (weight, id); leaves have
 *    id = symbol, the k-th merged node id 16 + k.  One symbol gets length 1.
 *  - length limit binds only below depth 15 (16 leaves): then package-merge
 *    (Larmore and Hirschberg 1990), leaves before packages on equal weight.
 *  - canonical code (RFC 1951 §3.2.2): codes in (length, symbol) order.
 *  - code order: the stream holds one code per weight, in weight order,
 *    except that inside every whole block of 8 weights (weights 8b..8b+7,
 *    all < n) the codes come in the order 8b+0, 8b+4, 8b+1, 8b+5, 8b+2,
 *    8b+6, 8b+3, 8b+7; a last block of fewer than 8 weights keeps weight
 *    order.  Code i of the stream is weight coded_weight(i).  ("Code i",
 *    as in the gaps and group offsets below, counts codes in stream order.)
 *  - code stream: little-endian 32-bit words, bit i of the stream is bit
 *    31 - (i mod 32) of word i / 32 (MSB first within a word).  Inside each
 *    group of T chunks the words are stored word-major: word m of chunk c at
 *    position m T + c of the group, so that the T threads of a group read
 *    their chunks' word m from adjacent words.
 *  - chunk c = stream bits [8Cc, 8C(c+1)); gap_c = first code start at or
 *    after 8Cc minus 8Cc, 4 bits per chunk (p1 §3.2.1 gap[tid]).  The end of
 *    the stream (bit code_bits) counts as a start, so a chunk that begins
 *    inside the last code points past it; chunks beyond the end hold 0.
 *  - group g = T chunks; off[g] = number of codes starting before bit 8CTg.
 *  - sign/mantissa nibbles, 8 weights per little-endian 32-bit word w: for
 *    k = 0..3, byte k holds weight 8w+k's sign in bit 7 and mantissa in bits
 *    0-2, weight 8w+4+k's mantissa in bits 4-6, and in bit 3 the sign of
 *    weight 8w+4+((k+3) mod 4), i.e. weight 8w+4+k's sign sits in bit 3 of
 *    byte (k+1) mod 4.  Four bits per weight, as the pages' nibble array.
 *  - no decode table in the blob: the code lengths in the header are the
 *    codebook, and a decoder derives whatever table it uses from them.
 *
 * Parity pins live in tests/test_oracle_pins.py.  Functions whose result has
 * no pin are marked "parity unpinned" (none at present).
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define NSYM 16
#define HEADER_BYTES 128
#define MAGIC 0x38464345u /* bytes 'E' 'C' 'F' '8' */
#define VERSION 3u

/* ---------- little-endian field access ---------- */
static uint32_t rd32(const uint8_t* p) {
  return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}
static uint64_t rd64(const uint8_t* p) { return (uint64_t)rd32(p) | ((uint64_t)rd32(p + 4) << 32); }
static void wr32(uint8_t* p, uint32_t v) {
  p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); p[2] = (uint8_t)(v >> 16); p[3] = (uint8_t)(v >> 24);
}
static void wr64(uint8_t* p, uint64_t v) { wr32(p, (uint32_t)v); wr32(p + 4, (uint32_t)(v >> 32)); }

/* ---------- step 1: split a byte (E4M3 = 1 sign, 4 exponent, 3 mantissa bits) ---------- */
int oracle_exponent(uint8_t b) { return (b >> 3) & 15; }
int oracle_nibble(uint8_t b) { return ((b >> 7) << 3) | (b & 7); }
uint8_t oracle_join(int e, int nib) { return (uint8_t)(((nib >> 3) << 7) | (e << 3) | (nib & 7)); }

/* ---------- step 2: exponent histogram (p1 §3.1.1 item 1, §5.1 collect_exp_stats) ---------- */
int oracle_histogram(const uint8_t* x, uint64_t n, uint64_t* hist) {
  for (int s = 0; s < NSYM; ++s) hist[s] = 0;
  for (uint64_t i = 0; i < n; ++i) hist[oracle_exponent(x[i])] += 1;
  return 0;
}

/* ---------- step 3: Huffman code lengths (p1 §3.1.1 item 2, build_huffman) ---------- */
int oracle_huffman_lengths(const uint64_t* hist, uint8_t* len) {
  uint64_t weight[2 * NSYM];
  int parent[2 * NSYM], alive[2 * NSYM];
  int nodes = 0, live = 0;
  for (int s = 0; s < NSYM; ++s) len[s] = 0;
  for (int s = 0; s < NSYM; ++s) {
    weight[s] = hist[s];
    parent[s] = -1;
    alive[s] = hist[s] > 0;
    live += alive[s];
  }
  nodes = NSYM;
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
    len[s] = (uint8_t)d;
  }
  return 0;
}

/* ---------- step 4: length-limited lengths by package-merge (p1 §3.1.1 item 3) ---------- */
typedef struct { uint64_t w; int is_leaf; int cnt[NSYM]; } pm_item;

static void pm_sort_leaves(pm_item* a, int k) { /* insertion sort by (weight, symbol) */
  for (int i = 1; i < k; ++i) {
    pm_item t = a[i];
    int j = i - 1;
    while (j >= 0 && a[j].w > t.w) { a[j + 1] = a[j]; --j; }
    a[j + 1] = t;
  }
}

int oracle_package_merge_lengths(const uint64_t* hist, int max_len, uint8_t* len) {
  pm_item leaves[NSYM];
  static pm_item list[4 * NSYM], next[4 * NSYM], pkg[2 * NSYM];
  int k = 0;
  for (int s = 0; s < NSYM; ++s) len[s] = 0;
  for (int s = 0; s < NSYM; ++s) {
    if (hist[s] == 0) continue;
    memset(&leaves[k], 0, sizeof(pm_item));
    leaves[k].w = hist[s];
    leaves[k].is_leaf = 1;
    leaves[k].cnt[s] = 1;
    k += 1;
  }
  if (k == 0) return 0;
  if (k == 1) { for (int s = 0; s < NSYM; ++s) if (hist[s]) len[s] = 1; return 0; }
  if (max_len < 1 || max_len > 16 || (1 << max_len) < k) return -1;
  pm_sort_leaves(leaves, k);
  int nl = k;
  for (int i = 0; i < k; ++i) list[i] = leaves[i];
  for (int level = 1; level < max_len; ++level) {
    int np = nl / 2;
    for (int i = 0; i < np; ++i) {
      pkg[i].w = list[2 * i].w + list[2 * i + 1].w;
      pkg[i].is_leaf = 0;
      for (int s = 0; s < NSYM; ++s) pkg[i].cnt[s] = list[2 * i].cnt[s] + list[2 * i + 1].cnt[s];
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

/* Plain Huffman unless it is deeper than max_len; then package-merge. */
int oracle_code_lengths(const uint64_t* hist, int max_len, uint8_t* len) {
  if (oracle_huffman_lengths(hist, len) != 0) return -1;
  int deepest = 0;
  for (int s = 0; s < NSYM; ++s) if (len[s] > deepest) deepest = len[s];
  if (deepest <= max_len) return 0;
  return oracle_package_merge_lengths(hist, max_len, len);
}

/* ---------- step 5: canonical codes (RFC 1951 §3.2.2) ---------- */
int oracle_canonical_codes(const uint8_t* len, uint32_t* code) {
  int count[18] = {0};
  uint32_t next[18] = {0};
  for (int s = 0; s < NSYM; ++s) {
    if (len[s] > 16) return -1;
    if (len[s]) count[len[s]] += 1;
  }
  uint32_t c = 0;
  for (int l = 1; l <= 16; ++l) {
    c = (c + (uint32_t)count[l - 1]) << 1;
    next[l] = c;
  }
  for (int s = 0; s < NSYM; ++s) code[s] = len[s] ? next[len[s]]++ : 0;
  return 0;
}

/* ---------- bit access: MSB first inside little-endian 32-bit words ---------- */
/* The stream section of a blob with its layout: chunks of C bytes, T chunks
 * per group. */
typedef struct { uint8_t* base; uint32_t C, T; } stream_t;

/* Byte offset of the 32-bit word that holds stream bit i.  Bit i lies in
 * word i / 32 of the stream read in order, which is word m of chunk c of
 * group g; inside a group the words are stored word-major, word m of chunk c
 * at position m * T + c, so the T chunks' word m sit side by side. */
static uint64_t word_offset(const stream_t* s, uint64_t i) {
  uint64_t w = i / 32, per_chunk = s->C / 4, per_group = per_chunk * s->T;
  uint64_t g = w / per_group, r = w % per_group;
  uint64_t c = r / per_chunk, m = r % per_chunk;
  return 4 * (g * per_group + m * s->T + c);
}

static int get_bit(const stream_t* s, uint64_t i) {
  uint32_t w = rd32(s->base + word_offset(s, i));
  return (int)((w >> (31 - (i % 32))) & 1u);
}
static void set_bit(stream_t* s, uint64_t i) {
  uint8_t* p = s->base + word_offset(s, i);
  wr32(p, rd32(p) | (1u << (31 - (i % 32))));
}

/* Match one code by reading bits one at a time; -1 if no code matches within
 * `avail` bits (or 16).  *used gets the code length. */
static int match_code(const uint8_t* len, const uint32_t* code, int (*bit)(const void*, uint64_t),
                      const void* src, uint64_t at, uint64_t avail, int* used) {
  uint32_t c = 0;
  for (int l = 1; l <= 16 && (uint64_t)l <= avail; ++l) {
    c = (c << 1) | (uint32_t)bit(src, at + (uint64_t)(l - 1));
    for (int s = 0; s < NSYM; ++s)
      if (len[s] == l && code[s] == c) { *used = l; return s; }
  }
  return -1;
}

static int stream_bit(const void* src, uint64_t i) { return get_bit((const stream_t*)src, i); }
/* The weight whose exponent is code i of the stream (see the code order
 * above): position r = i mod 8 of a whole block holds weight r / 2 of the
 * block's first half when r is even, weight 4 + r / 2 of its second half
 * when r is odd. */
static uint64_t coded_weight(uint64_t i, uint64_t n) {
  uint64_t block = i / 8, r = i % 8;
  if (8 * block + 8 > n) return i; /* the last, partial block */
  return 8 * block + (r % 2 == 0 ? r / 2 : 4 + r / 2);
}

/* ---------- blob layout ---------- */
typedef struct {
  uint64_t n, code_bits, groups;
  uint32_t C, T;
  uint64_t gaps_off, gaps_size, groups_off, groups_size;
  uint64_t stream_off, stream_size, nib_off, nib_size, total;
} layout_t;

static uint64_t up256(uint64_t x) { return (x + 255) / 256 * 256; }

static int make_layout(uint64_t n, uint64_t code_bits, uint32_t C, uint32_t T, layout_t* L) {
  if (C < 4 || C % 4 != 0 || T < 1) return -1;
  memset(L, 0, sizeof(*L));
  L->n = n; L->code_bits = code_bits; L->C = C; L->T = T;
  uint64_t group_bits = 8ull * C * T;
  L->groups = (code_bits + group_bits - 1) / group_bits;
  uint64_t chunks = L->groups * T;
  L->gaps_size = (chunks + 7) / 8 * 4;
  L->gaps_size = (L->gaps_size + 15) / 16 * 16;
  L->groups_size = 8 * (L->groups + 1);
  L->stream_size = n ? L->groups * T * C + 16 : 0;
  L->nib_size = (n + 31) / 32 * 16;
  L->gaps_off = up256(HEADER_BYTES);
  L->groups_off = up256(L->gaps_off + L->gaps_size);
  L->stream_off = up256(L->groups_off + L->groups_size);
  L->nib_off = up256(L->stream_off + L->stream_size);
  L->total = L->nib_off + L->nib_size;
  return 0;
}

static uint64_t total_code_bits(const uint8_t* x, uint64_t n, const uint8_t* len) {
  uint64_t bits = 0;
  for (uint64_t i = 0; i < n; ++i) bits += len[oracle_exponent(x[i])];
  return bits;
}

uint64_t oracle_encoded_size(const uint8_t* x, uint64_t n, const uint8_t* len, uint32_t C, uint32_t T) {
  layout_t L;
  if (make_layout(n, total_code_bits(x, n, len), C, T, &L) != 0) return 0;
  return L.total;
}

/* ---------- step 6-9: encode (bit-serial writer) ---------- */
int oracle_encode(const uint8_t* x, uint64_t n, const uint8_t* len, uint32_t C, uint32_t T,
                  uint8_t* blob, uint64_t cap, uint64_t* size) {
  uint32_t code[NSYM];
  int max_len = 0;
  for (int s = 0; s < NSYM; ++s) if (len[s] > max_len) max_len = len[s];
  if (max_len > 16 || oracle_canonical_codes(len, code) != 0) return -1;
  for (uint64_t i = 0; i < n; ++i)
    if (len[oracle_exponent(x[i])] == 0) return -2; /* exponent without a code */
  layout_t L;
  if (make_layout(n, total_code_bits(x, n, len), C, T, &L) != 0) return -1;
  if (cap < L.total) return -3;
  memset(blob, 0, L.total);

  /* header */
  wr32(blob + 0, MAGIC);
  wr32(blob + 4, VERSION);
  wr64(blob + 8, n);
  wr64(blob + 16, L.code_bits);
  wr32(blob + 24, C);
  wr32(blob + 28, T);
  wr32(blob + 32, (uint32_t)L.groups);
  wr32(blob + 36, 0); /* reserved */
  wr32(blob + 40, (uint32_t)max_len);
  wr32(blob + 44, HEADER_BYTES);
  wr64(blob + 48, 0); /* reserved */
  wr64(blob + 56, L.gaps_off);
  wr64(blob + 64, L.groups_off);
  wr64(blob + 72, L.stream_off);
  wr64(blob + 80, L.nib_off);
  wr64(blob + 88, L.total);
  for (int s = 0; s < NSYM; ++s) blob[96 + s] = len[s];

  /* code stream, one bit at a time, and the code start positions it implies */
  stream_t stream = {blob + L.stream_off, C, T};
  uint8_t* gaps = blob + L.gaps_off;
  uint8_t* offs = blob + L.groups_off;
  uint64_t chunk_bits = 8ull * C, chunks = L.groups * T;
  uint64_t next_chunk = 0;  /* first chunk whose gap is not yet known */
  uint64_t pos = 0;
  for (uint64_t i = 0; i <= n; ++i) {
    /* every chunk that starts at or before this code's start, and after the
     * previous code's start, has this code as its first code; i == n is the
     * end of the stream */
    while (next_chunk < chunks && next_chunk * chunk_bits <= pos) {
      uint64_t gap = pos - next_chunk * chunk_bits;
      if (gap > 15) return -4;
      uint8_t* gp = gaps + 4 * (next_chunk / 8);
      wr32(gp, rd32(gp) | ((uint32_t)gap << (4 * (next_chunk % 8))));
      if (next_chunk % T == 0) wr64(offs + 8 * (next_chunk / T), i);
      next_chunk += 1;
    }
    if (i == n) break;
    int e = oracle_exponent(x[coded_weight(i, n)]);
    for (int b = len[e] - 1; b >= 0; --b) {
      if ((code[e] >> b) & 1u) set_bit(&stream, pos);
      pos += 1;
    }
  }
  /* chunks wholly past the end keep gap 0; their groups start at n */
  for (; next_chunk < chunks; ++next_chunk)
    if (next_chunk % T == 0) wr64(offs + 8 * (next_chunk / T), n);
  wr64(offs + 8 * L.groups, n);

  /* sign + mantissa nibbles, bit by bit at the places the layout gives them */
  uint8_t* nib = blob + L.nib_off;
  for (uint64_t i = 0; i < n; ++i) {
    int v = oracle_nibble(x[i]);
    int sign = (v >> 3) & 1, mant = v & 7;
    uint64_t word = 4 * (i / 8);
    int r = (int)(i % 8);
    if (r < 4) {
      nib[word + r] |= (uint8_t)((sign << 7) | mant);
    } else {
      int k = r - 4;
      nib[word + k] |= (uint8_t)(mant << 4);
      nib[word + (k + 1) % 4] |= (uint8_t)(sign << 3);
    }
  }
  *size = L.total;
  return 0;
}

/* ---------- header parse ---------- */
static int read_layout(const uint8_t* blob, uint64_t size, layout_t* L, uint8_t* len) {
  if (size < HEADER_BYTES || rd32(blob) != MAGIC || rd32(blob + 4) != VERSION) return -1;
  if (rd32(blob + 36) != 0 || rd32(blob + 44) != HEADER_BYTES) return -1;
  uint64_t n = rd64(blob + 8), code_bits = rd64(blob + 16);
  if (make_layout(n, code_bits, rd32(blob + 24), rd32(blob + 28), L) != 0) return -1;
  if (L->groups != rd32(blob + 32) || rd64(blob + 48) != 0 || L->gaps_off != rd64(blob + 56) ||
      L->groups_off != rd64(blob + 64) || L->stream_off != rd64(blob + 72) ||
      L->nib_off != rd64(blob + 80) || L->total != rd64(blob + 88) || L->total > size)
    return -1;
  for (int s = 0; s < NSYM; ++s) len[s] = blob[96 + s];
  return 0;
}

/* ---------- step 10: bit-serial decode; ignores gaps and offsets ---------- */
int oracle_decode(const uint8_t* blob, uint64_t size, uint8_t* out, uint64_t n) {
  layout_t L;
  uint8_t len[NSYM];
  uint32_t code[NSYM];
  if (read_layout(blob, size, &L, len) != 0) return -1;
  if (n != L.n) return -2;
  if (oracle_canonical_codes(len, code) != 0) return -1;
  const stream_t stream = {(uint8_t*)(blob + L.stream_off), L.C, L.T};
  const uint8_t* nib = blob + L.nib_off;
  uint64_t pos = 0;
  for (uint64_t i = 0; i < n; ++i) {
    int used = 0;
    int e = match_code(len, code, stream_bit, &stream, pos, L.code_bits - pos, &used);
    if (e < 0) return -5;
    pos += (uint64_t)used;
    const uint64_t w = coded_weight(i, n); /* code i is this weight's exponent */
    const uint8_t* word = nib + 4 * (w / 8);
    int r = (int)(w % 8), sign, mant;
    if (r < 4) {
      sign = (word[r] >> 7) & 1;
      mant = word[r] & 7;
    } else {
      mant = (word[r - 4] >> 4) & 7;
      sign = (word[(r - 3) % 4] >> 3) & 1;
    }
    out[w] = oracle_join(e, (sign << 3) | mant);
  }
  return pos == L.code_bits ? 0 : -6;
}

/* ---------- recompute gaps and group offsets by the serial walk ---------- */
int oracle_check_index(const uint8_t* blob, uint64_t size) {
  layout_t L;
  uint8_t len[NSYM];
  uint32_t code[NSYM];
  if (read_layout(blob, size, &L, len) != 0) return -1;
  if (oracle_canonical_codes(len, code) != 0) return -1;
  const stream_t stream = {(uint8_t*)(blob + L.stream_off), L.C, L.T};
  uint64_t chunk_bits = 8ull * L.C, chunks = L.groups * L.T, c = 0, pos = 0;
  for (uint64_t i = 0; i <= L.n + 1; ++i) {
    /* code starts, then the end of the stream, then a start past every chunk */
    uint64_t start = i < L.n ? pos : (i == L.n ? L.code_bits : UINT64_MAX);
    while (c < chunks && c * chunk_bits <= start) {
      uint32_t want = i <= L.n ? (uint32_t)(start - c * chunk_bits) : 0;
      uint32_t got = (rd32(blob + L.gaps_off + 4 * (c / 8)) >> (4 * (c % 8))) & 15u;
      if (got != want) return 2;
      uint64_t first = i < L.n ? i : L.n;
      if (c % L.T == 0 && rd64(blob + L.groups_off + 8 * (c / L.T)) != first) return 3;
      c += 1;
    }
    if (i >= L.n) continue;
    int used = 0;
    if (match_code(len, code, stream_bit, &stream, pos, L.code_bits - pos, &used) < 0) return 4;
    pos += (uint64_t)used;
  }
  if (rd64(blob + L.groups_off + 8 * L.groups) != L.n) return 3;
  return 0;
}
