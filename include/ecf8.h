/*
 * ecf8.h -- C ABI of the ECF8 (Exponent-Concentrated FP8) lossless codec for
 * FP8 E4M3 weight tensors: host-side encoder and sm_100a GPU decoder.
 *
 * Method ("To Compress or Not? Pushing the Frontier of Lossless GenAI Model
 * Weights Compression with Exponent Concentration", arXiv 2510.02676,
 * abstract; ECF8 walkthrough "ECF8 浮点数压缩技术" §3.1-§3.2): the 4-bit exponent
 * field of every E4M3 weight is coded with a per-tensor canonical Huffman
 * code of at most 16 bits, sign and mantissa are kept raw as a nibble array,
 * and decoding reproduces every original byte exactly.
 *
 * Conventions for every call:
 *  - Return value: ECF8_OK (0) or a negative ECF8_ERR_* code; ecf8_strerror
 *    names it.  No call throws, aborts or prints.
 *  - The caller owns every buffer, host and device.  Between calls the
 *    library keeps per-device kernel attributes (set once), a launch counter,
 *    and one device table of its own: ECF8_NOALLOC_MAX_TENSORS descriptors of
 *    96 bytes on every GPU that loads the library, used only by
 *    ecf8_decode_batched_noalloc, overwritten by each such call and held until
 *    the process exits.  No call allocates device memory.
 *  - "host" pointers are ordinary CPU memory; "device" pointers are CUDA
 *    global memory of the current device and must be 16-byte aligned.
 *  - Decode calls are asynchronous on the given stream.  Argument and header
 *    errors are returned before anything is enqueued.  Corrupt data found by
 *    the kernel is reported by OR-ing ECF8_STATUS_* bits into *d_status
 *    (device int32, nullable), which the caller reads after synchronising.
 *    The kernels never read outside [d_blob, d_blob + blob_size), never write
 *    outside [d_out, d_out + n) and never wait.
 *
 * Blob layout (version 3, all fields little-endian; the on-disk and in-HBM
 * form of one compressed tensor):
 *   header, 128 bytes:
 *     0 u32 magic 0x38464345 ("ECF8")   4 u32 version = 3
 *     8 u64 n (weights)                16 u64 code_bits (stream length in bits)
 *    24 u32 chunk_bytes C              28 u32 group_chunks T
 *    32 u32 n_groups G                 36 u32 reserved = 0
 *    40 u32 max code length            44 u32 header bytes = 128
 *    48 u64 reserved = 0               56 u64 offset of gaps
 *    64 u64 offset of group offsets    72 u64 offset of code stream
 *    80 u64 offset of nibbles          88 u64 blob bytes
 *    96 u8[16] code length per exponent value (0 = absent)   112 u8[16] zero
 *   code order: one code per weight; inside every whole block of 8 weights
 *     (8b..8b+7 < n) the codes come in the order 8b+0, 8b+4, 8b+1, 8b+5,
 *     8b+2, 8b+6, 8b+3, 8b+7, and a last block of fewer than 8 weights keeps
 *     weight order.  "Code i" below counts codes in this stream order.
 *   sections, each at a multiple of 256 bytes, in this order:
 *     gaps          4 bits per chunk, chunk c in bits 4(c%8) of u32 word c/8;
 *                   offset of the first code start at or after the chunk start
 *                   (the stream end counts as a start), 0 past the end.
 *     group offsets G+1 u64: number of codes starting before bit 8*C*T*g.
 *     code stream   G*T*C bytes + 16 zero bytes of u32 words.  Stream bit i
 *                   is bit 31-(i%32) of reading-order word i/32; inside each
 *                   group of T chunks, reading-order word m of chunk c is
 *                   stored at word m*T + c of the group (word-major), so the
 *                   T decoder threads' word m are adjacent.
 *     nibbles       ceil(n/32)*16 bytes, 8 weights per u32 word w: byte k
 *                   (k = 0..3) holds weight 8w+k's sign in bit 7 and mantissa
 *                   in bits 0-2, weight 8w+4+k's mantissa in bits 4-6, and in
 *                   bit 3 the sign of weight 8w+4+((k+3)%4).
 * The 16 code lengths are the whole codebook: the canonical code follows from
 * them, and the decoder builds its tables from them.
 */
#ifndef ECF8_H_
#define ECF8_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h> /* cudaStream_t */

#ifdef __cplusplus
extern "C" {
#endif

#define ECF8_ABI_VERSION 2

/* return codes */
#define ECF8_OK 0
#define ECF8_ERR_ARG (-1)         /* null pointer, bad size or parameter */
#define ECF8_ERR_FORMAT (-2)      /* blob header or layout inconsistent */
#define ECF8_ERR_CAPACITY (-3)    /* destination buffer too small */
#define ECF8_ERR_CODEBOOK (-4)    /* invalid code lengths, or an exponent with no code */
#define ECF8_ERR_ALIGN (-5)       /* device pointer not 16-byte aligned */
#define ECF8_ERR_UNSUPPORTED (-6) /* layout the GPU kernels do not implement */
#define ECF8_ERR_CUDA (-7)        /* a CUDA runtime call failed */
#define ECF8_ERR_WORKSPACE (-8)   /* workspace null or too small */
#define ECF8_ERR_TOO_MANY (-9)    /* more tensors than ecf8_decode_batched_noalloc holds */
#define ECF8_ERR_CAPTURE (-10)    /* a call that copies from host memory was made while its stream captures */

/* bits OR-ed into *d_status by the decode kernels */
#define ECF8_STATUS_COUNT_MISMATCH 1 /* codes decoded in a group != its offset delta */
#define ECF8_STATUS_BAD_CODE 2       /* bits that match no code */
#define ECF8_STATUS_BAD_OFFSETS 4    /* group offsets not monotone or past n */
#define ECF8_STATUS_BOUNDS 8         /* checked builds only: an index failed its bounds check */

/* A canonical Huffman code over the 16 exponent values. */
typedef struct ecf8_codebook {
  uint8_t len[16];   /* code length in bits, 0 = value absent */
  uint16_t code[16]; /* canonical code, right-aligned, valid where len > 0 */
  uint32_t max_len;  /* longest length present */
  uint32_t n_symbols;
} ecf8_codebook;

/* Header of one blob, as read on the host by ecf8_blob_info.  Decode calls
 * take it so that they never read the device blob back. */
typedef struct ecf8_info {
  uint64_t n;
  uint64_t code_bits;
  uint64_t blob_bytes;
  uint64_t gaps_off, groups_off, stream_off, nibbles_off;
  uint32_t chunk_bytes;
  uint32_t group_chunks;
  uint32_t n_groups;
  uint32_t max_len;
  uint8_t len[16];
} ecf8_info;

/* One tensor of a batched decode. */
typedef struct ecf8_tensor {
  const ecf8_info* info; /* host */
  const void* d_blob;    /* device, 16-byte aligned */
  size_t blob_size;      /* bytes readable at d_blob; at least info->blob_bytes */
  uint8_t* d_out;        /* device, 16-byte aligned, info->n bytes */
} ecf8_tensor;

/* Exponent histogram of n E4M3 bytes (ECF8 walkthrough §3.1.1 step 1,
 * §5.1 collect_exp_stats).  host in, host out. */
int ecf8_histogram(const uint8_t* fp8, size_t n, uint64_t hist[16]);

/* Optimal prefix code of at most max_len bits (1..16) for a histogram (§3.1.1
 * steps 2-3, build_huffman).  Huffman with ties broken by (weight, node id),
 * leaves numbered by value and merged nodes 16, 17, ...; when that tree is
 * deeper than max_len, package-merge.  A single present value gets a 1-bit
 * code.  ECF8_ERR_CODEBOOK when 2^max_len < number of present values. */
int ecf8_build_codebook(const uint64_t hist[16], uint32_t max_len, ecf8_codebook* out);

/* Exact blob size for n weights with histogram hist under cb (the
 * compressed size the ECF8 walkthrough §3.1.1 reports as the memory saving:
 * code bits from the histogram, plus the per-chunk and per-group metadata of
 * §3.2.1 and the raw sign/mantissa nibbles).  host.  ECF8_ERR_CODEBOOK if an
 * exponent in hist has no code; ECF8_ERR_ARG on a bad layout or when the
 * histogram does not sum to n. */
int ecf8_encoded_size(const uint64_t hist[16], size_t n, const ecf8_codebook* cb,
                      uint32_t chunk_bytes, uint32_t group_chunks, size_t* out_bytes);

/* An upper bound on the blob size of ANY n weights under any code of at most
 * 16 bits, with this layout, that needs no histogram (for sizing a buffer
 * before the weights are seen).  0 for an invalid layout or an n so large the
 * bound overflows. */
size_t ecf8_encoded_size_bound(size_t n, uint32_t chunk_bytes, uint32_t group_chunks);

/* Encode n E4M3 bytes into blob (host, capacity cap): the ECF8 walkthrough
 * §3.1.1 steps (exponent field coded with cb, sign and mantissa kept raw)
 * and the per-thread metadata of §3.2.1, in the version-3 layout above.
 * chunk_bytes is the stream slice of one decoder thread (multiple of 4),
 * group_chunks the chunks that share one group offset.  ECF8_ERR_CODEBOOK if
 * a present exponent has no code or cb's codes are not the canonical code of
 * its lengths; ECF8_ERR_CAPACITY if cap is short.  *blob_bytes gets the size.
 * Multi-threaded over ranges of >= 1M weights; the bytes do not depend on the
 * thread count. */
int ecf8_encode(const uint8_t* fp8, size_t n, const ecf8_codebook* cb, uint32_t chunk_bytes,
                uint32_t group_chunks, void* blob, size_t cap, size_t* blob_bytes);

/* Parse and check a blob's header (the metadata a decoder of the ECF8
 * walkthrough §3.2.1 is given beside the bitstream): magic, version, the
 * section layout against n, code_bits, C and T, and the code lengths (a
 * prefix code of at most 16 bits, Kraft sum <= 1).  blob (host) must hold at
 * least the 128-byte header, which is all the call reads; size is the number
 * of bytes the whole blob occupies where it is stored (host or device), and
 * must cover the layout's total.  ECF8_ERR_FORMAT, ECF8_ERR_CODEBOOK. */
int ecf8_blob_info(const void* blob, size_t size, ecf8_info* out);

/* 1 if the GPU kernels implement (chunk_bytes, group_chunks), else 0. */
int ecf8_layout_supported(uint32_t chunk_bytes, uint32_t group_chunks);

/* Decode one tensor on the GPU (ECF8 walkthrough §3.2.1, decode_kernel over
 * the bitstream and its metadata): d_blob (device copy of the blob described
 * by info, blob_size bytes readable) -> d_out (n bytes).  n must equal
 * info->n and blob_size must be at least info->blob_bytes (ECF8_ERR_ARG
 * otherwise, before anything is enqueued).  One kernel launch on stream s; no
 * launch when n = 0. */
int ecf8_decode(const ecf8_info* info, const void* d_blob, size_t blob_size, uint8_t* d_out, size_t n,
                int32_t* d_status, cudaStream_t s);

/* Batches of at most this many tensors need no workspace. */
#define ECF8_BATCH_INLINE_MAX 64

/* Bytes of device workspace ecf8_decode_batched needs for count tensors
 * (0 when count <= ECF8_BATCH_INLINE_MAX). */
size_t ecf8_batched_workspace_size(int count);

/* Decode count tensors in ONE kernel launch (batching across tensors as in
 * the DFloat11 article's block-level batching, §3.3).  All tensors must share
 * chunk_bytes and group_chunks; each tensor's blob_size must cover its
 * info->blob_bytes (ECF8_ERR_ARG).  Up to ECF8_BATCH_INLINE_MAX tensors travel
 * in the launch's parameter block and d_workspace may be NULL.  Larger batches
 * copy a descriptor table from host memory into d_workspace (device, 16-byte
 * aligned) on stream s before the launch; the workspace must not be touched by
 * other streams until the decode ends.  That copy reads a temporary host
 * array, so such a call returns ECF8_ERR_CAPTURE, enqueueing nothing, while s
 * is capturing a CUDA graph; batches of up to ECF8_BATCH_INLINE_MAX tensors
 * copy nothing from the host. */
int ecf8_decode_batched(const ecf8_tensor* tensors, int count, void* d_workspace, size_t workspace_bytes,
                        int32_t* d_status, cudaStream_t s);

/* Most tensors one ecf8_decode_batched_noalloc call takes. */
#define ECF8_NOALLOC_MAX_TENSORS 1024

/* ecf8_decode_batched without a workspace, for callers that cannot allocate
 * device memory when they decode: for example a plugin running inside an
 * inference engine that owns every device allocation and hands out no
 * scratch, or a serving loop that must not call cudaMalloc because it
 * synchronises the device and can stall other streams.  The paper has no
 * counterpart of this call; it is a property of this library.
 *
 * The descriptor table that ecf8_decode_batched copies into the caller's
 * workspace goes instead into one table in device memory that the library
 * itself holds: ECF8_NOALLOC_MAX_TENSORS entries of 96 bytes (96 KB) on
 * every GPU that loads the library, kept until the process exits.  The caller
 * still provides every blob and output buffer.  The call makes no cudaMalloc,
 * cudaFree or other allocating call.
 *  - The first call on a device resolves that table's device address (and
 *    sets the kernel attributes); make that first call before any stream
 *    capture.
 *  - Every call on a device shares the one table and overwrites it.  Calls
 *    ordered on one stream are fine; calls that can overlap on the GPU
 *    (different streams without ordering between them) race and may decode
 *    with each other's descriptors.
 *  - count > ECF8_NOALLOC_MAX_TENSORS returns ECF8_ERR_TOO_MANY and enqueues
 *    nothing.  Other arguments and errors are as for ecf8_decode_batched. */
int ecf8_decode_batched_noalloc(const ecf8_tensor* tensors, int count, int32_t* d_status, cudaStream_t s);

/* ---------------------------------------------------------------------------
 * Encoding on the GPU (the same blob as ecf8_encode, byte for byte).  The
 * histogram and every per-weight step run in kernels; the 16-symbol code and
 * the header/decode-table prefix are built on the host.
 *   ecf8_histogram_device(d_x, n, d_hist, s);          -- device counts
 *   copy d_hist to the host, ecf8_build_codebook(hist, 16, &cb);
 *   ecf8_encoded_size(hist, n, &cb, C, T, &bytes);      -- blob size
 *   ecf8_encode_device(d_x, n, hist, &cb, C, T, d_blob, bytes, &bytes, ws, ws_bytes, s);
 * d_fp8, d_hist, d_blob and the workspace are device memory, 16-byte aligned.
 */

/* Exponent histogram of n E4M3 bytes in device memory into d_hist[16]
 * (device, uint64; zeroed by the call).  Asynchronous on stream s. */
int ecf8_histogram_device(const uint8_t* d_fp8, size_t n, uint64_t* d_hist, cudaStream_t s);

/* Bytes of device workspace ecf8_encode_device needs for n weights. */
size_t ecf8_encode_device_workspace_size(size_t n);

/* Encode n E4M3 bytes in device memory into d_blob (device, blob_cap bytes):
 * the blob ecf8_encode writes for the same input, codebook and layout.
 * hist (host) is the input's exponent histogram, which fixes the blob's size;
 * cb must give every exponent that occurs a code (ECF8_ERR_CODEBOOK
 * otherwise).  Asynchronous on stream s; *blob_bytes is set on return.
 * Errors: ECF8_ERR_ARG, ECF8_ERR_ALIGN, ECF8_ERR_CODEBOOK, ECF8_ERR_CAPACITY,
 * ECF8_ERR_WORKSPACE, ECF8_ERR_CUDA. */
int ecf8_encode_device(const uint8_t* d_fp8, size_t n, const uint64_t hist[16], const ecf8_codebook* cb,
                       uint32_t chunk_bytes, uint32_t group_chunks, void* d_blob, size_t blob_cap,
                       size_t* blob_bytes, void* d_workspace, size_t workspace_bytes, cudaStream_t s);

/* ecf8_decode_batched with the persistent grid capped at max_ctas CTAs (one
 * CTA occupies a whole SM's shared memory), so that a decode running beside
 * other kernels leaves them the remaining SMs.  max_ctas = 0: one CTA per SM.
 * A batch that mixes tensors with and without a 1-bit code takes at least 2. */
int ecf8_decode_batched_ctas(const ecf8_tensor* tensors, int count, void* d_workspace, size_t workspace_bytes,
                             int32_t* d_status, cudaStream_t s, uint32_t max_ctas);

/* ---------------------------------------------------------------------------
 * Decode-on-use pipeline (ECF8 walkthrough §3.2.2 "即用即解压": a pool sized
 * for the largest layer, the layer's forward pass triggers its decode, the
 * pool is reused cyclically with no allocation; DFloat11 article §4: decode
 * the next layers in the background while the current one computes).
 *
 * Layer m is decoded into slot m % n_slots on decode_stream, `depth` layers
 * ahead of the one the compute stream asks for, once the compute stream has
 * released that slot's previous layer.  Protocol per layer, in any order of
 * layers (a forward pass takes them in order, and a new pass may start again
 * at layer 0):
 *     ecf8_pipeline_acquire(p, l, compute, &w);   -- compute waits for l
 *     ... kernels on `compute` read layer l's FP8 weights at w ...
 *     ecf8_pipeline_release(p, l, compute);       -- the slot may be reused
 * n_slots must be at least depth + 1 (the slot being decoded ahead is never
 * the one in use).  A layer still resident in its slot is not decoded again.
 */
typedef struct ecf8_layer_tensor {
  const ecf8_info* info; /* host; copied at create time */
  const void* d_blob;    /* device, 16-byte aligned, stays valid while the pipeline lives */
  size_t blob_size;      /* bytes readable at d_blob; at least info->blob_bytes */
  size_t out_offset;     /* byte offset of its FP8 output within a slot; multiple of 16 (of 32 for
                            the fastest stores); out_offset + info->n <= slot_bytes */
} ecf8_layer_tensor;

typedef struct ecf8_layer {
  const ecf8_layer_tensor* tensors; /* host; copied at create time */
  int count;
} ecf8_layer;

typedef struct ecf8_pipeline ecf8_pipeline; /* opaque */

/* Creates a pipeline over n_layers layers and n_slots caller-owned device
 * buffers of slot_bytes each (16-byte aligned).  d_workspace (device) is
 * needed only when a layer has more than ECF8_BATCH_INLINE_MAX tensors
 * (ecf8_batched_workspace_size of the largest layer); d_status (device) gets
 * the decodes' status bits.  max_ctas caps each decode's grid (0: one CTA
 * per SM).  The pipeline creates two CUDA events per slot and allocates no
 * device memory.  Errors: ECF8_ERR_ARG (counts, depth, slot too small),
 * ECF8_ERR_ALIGN, ECF8_ERR_WORKSPACE, ECF8_ERR_CUDA. */
int ecf8_pipeline_create(const ecf8_layer* layers, int n_layers, void* const* d_slots, int n_slots,
                         size_t slot_bytes, int depth, uint32_t max_ctas, void* d_workspace,
                         size_t workspace_bytes, int32_t* d_status, cudaStream_t decode_stream,
                         ecf8_pipeline** out);

/* Makes stream `compute` wait until layer's weights are decoded, enqueues the
 * decodes of the next `depth` layers whose slots are free, and returns the
 * layer's slot in *d_weights.  Returns ECF8_ERR_ARG if the layer's slot still
 * holds another layer that has not been released. */
int ecf8_pipeline_acquire(ecf8_pipeline* p, int layer, cudaStream_t compute, void** d_weights);

/* Records, on `compute`, that the kernels reading layer's slot have been
 * enqueued; a later decode into that slot waits for them. */
int ecf8_pipeline_release(ecf8_pipeline* p, int layer, cudaStream_t compute);

/* Frees the pipeline's events and host state (work already enqueued still
 * runs to completion). */
void ecf8_pipeline_destroy(ecf8_pipeline* p);

/* Number of decode kernels this library has launched in this process. */
uint64_t ecf8_launch_count(void);

const char* ecf8_strerror(int code);
int ecf8_abi_version(void);


/* ---- BF16 variant (DFloat11 article §2-§3) --------------------------------
 * A BF16 weight x splits into its 8-bit exponent field (x >> 7) & 0xFF, which
 * is Huffman-coded per tensor over 256 values with codes of at most 16 bits,
 * and one kept byte (sign << 7) | mantissa, stored verbatim.  The blob reuses
 * the ECF8 stream, gap and group-offset layout; byte layout (little-endian):
 *   0 magic "DF11" (0x31314644), 4 version 1, 8 n, 16 code_bits, 24 chunk
 *   bytes, 28 group chunks, 32 groups, 36 max_len, 40 lens_off, 48 gaps_off,
 *   56 groups_off, 64 stream_off, 72 kept_off, 80 total bytes; sections at
 *   256-byte boundaries: 256 code lengths, 4-bit gaps (16-byte padded),
 *   groups + 1 u64 offsets, stream (+16 zero bytes), n kept bytes (padded to
 *   16). */
typedef struct ecf8_bf16_info {
  uint64_t n;
  uint64_t code_bits;
  uint64_t blob_bytes;
  uint64_t lens_off, gaps_off, groups_off, stream_off, kept_off;
  uint32_t chunk_bytes;
  uint32_t group_chunks;
  uint32_t n_groups;
  uint32_t max_len;
  uint8_t len[256];
} ecf8_bf16_info;

/* Code lengths (<= max_len, 1..16) for the exponents of n BF16 bit patterns:
 * Huffman with (weight, id) ties, package-merge when deeper than max_len; a
 * single present exponent gets a 1-bit code.  host in, host out. */
int ecf8_bf16_code_lengths(const uint16_t* x, size_t n, uint32_t max_len, uint8_t len[256]);

/* Exact blob size for x under len.  ECF8_ERR_CODEBOOK if an exponent of x has
 * no code, or if len is not a complete prefix code of at most 16 bits (a
 * single present value may have any length). */
int ecf8_bf16_encoded_size(const uint16_t* x, size_t n, const uint8_t len[256], uint32_t chunk_bytes,
                           uint32_t group_chunks, size_t* bytes);

/* Encode n BF16 bit patterns into blob (host, capacity cap; OpenMP threads
 * over ranges of >= 1M weights); the bytes are those of the oracle's encoder
 * for the same lengths, whatever the thread count.  ECF8_ERR_CODEBOOK as
 * for ecf8_bf16_encoded_size; ECF8_ERR_CAPACITY if cap is short; *bytes gets
 * the size. */
int ecf8_bf16_encode(const uint16_t* x, size_t n, const uint8_t len[256], uint32_t chunk_bytes,
                     uint32_t group_chunks, void* blob, size_t cap, size_t* bytes);

/* Parse and validate a BF16 blob header (host memory, size bytes):
 * ECF8_ERR_FORMAT on a bad magic, version or layout, ECF8_ERR_CODEBOOK on
 * code lengths that are not a complete prefix code. */
int ecf8_bf16_blob_info(const void* blob, size_t size, ecf8_bf16_info* out);

/* Bytes of the decode table (32768): 256 tree nodes x 16 nibbles, 8 bytes an
 * entry. */
size_t ecf8_bf16_table_bytes(void);

/* Fill h_table (host, ecf8_bf16_table_bytes() bytes) with the nibble-state
 * table of info's code: 256 nodes x 16 nibbles of two u32 words; entry
 * (node, nibble) at index node * 16 + nibble holds the exponents whose codes
 * end inside the nibble (8 bits each, first lowest) and (next node << 7) |
 * (8 x their count) << 16.  Node 0 is the root; node ecf8_bf16_table_nodes()
 * is the error node, which every invalid bit sequence reaches and never
 * leaves.  Copy it to the device once per codebook. */
int ecf8_bf16_build_table(const ecf8_bf16_info* info, void* h_table);

/* Number of tree nodes of info's code (the decoder reads the table's first
 * nodes + 1 nodes); 0 when the code lengths are not a valid code. */
uint32_t ecf8_bf16_table_nodes(const ecf8_bf16_info* info);

/* Decode one BF16 blob on the GPU.  d_blob (device, 16-byte aligned) holds
 * info->blob_bytes; d_table (device, 16-byte aligned) the table of
 * ecf8_bf16_build_table for the same info; d_out (device, 16-byte aligned)
 * gets n uint16 BF16 bit patterns.  Requires chunk_bytes 32 and group_chunks
 * 32 (ECF8_ERR_UNSUPPORTED otherwise).  Enqueued on stream; corrupt input
 * ORs ECF8_STATUS_* bits into *d_status (may be null) and leaves the group's
 * output unwritten. */
int ecf8_bf16_decode(const ecf8_bf16_info* info, const void* d_blob, const void* d_table, uint16_t* d_out, size_t n,
                     int32_t* d_status, cudaStream_t stream);

/* Table layouts of the BF16 decoder.  WIDE: 64-bit (node, nibble) entries,
 * any code.  NARROW: 32-bit (node, nibble) entries, codes of >= 2 bits.
 * NARROW_LANE: NARROW copied once per lane (bank-conflict free), codes of
 * >= 2 bits on at most 31 tree nodes.  BYTE: 64-bit (node, byte) entries,
 * half the steps, codes of >= 2 bits on at most 31 tree nodes.  AUTO: WIDE
 * when a 1-bit code exists, else BYTE when it holds, else NARROW. */
#define ECF8_BF16_LAYOUT_AUTO (-1)
#define ECF8_BF16_LAYOUT_WIDE 0
#define ECF8_BF16_LAYOUT_NARROW 1
#define ECF8_BF16_LAYOUT_NARROW_LANE 2
#define ECF8_BF16_LAYOUT_BYTE 3

/* One tensor of a batched BF16 decode (pointers as for ecf8_bf16_decode). */
typedef struct ecf8_bf16_tensor {
  const ecf8_bf16_info* info; /* host */
  const void* d_blob;         /* device, 16-byte aligned */
  const void* d_table;        /* device, 16-byte aligned, ecf8_bf16_build_table of info */
  uint16_t* d_out;            /* device, 16-byte aligned, info->n elements */
} ecf8_bf16_tensor;

/* Tensors a batched launch carries in its parameters. */
#define ECF8_BF16_BATCH_MAX 32

/* Decode count BF16 blobs: one launch per table layout present (AUTO per
 * tensor) and per ECF8_BF16_BATCH_MAX tensors, each CTA over a contiguous
 * run of the tensors' groups.  Every tensor is checked before anything is
 * enqueued (argument errors as ecf8_bf16_decode); empty tensors are skipped.
 * A CUDA error from a launch (ECF8_ERR_CUDA) can come after earlier launches
 * of the same call were enqueued: some outputs may then be decoded and others
 * not. */
int ecf8_bf16_decode_batched(const ecf8_bf16_tensor* tensors, int count, int32_t* d_status, cudaStream_t stream);

/* The layout ecf8_bf16_decode picks for info's code (>= 0), or an error. */
int ecf8_bf16_auto_layout(const ecf8_bf16_info* info);

/* ecf8_bf16_decode with a given table layout; ECF8_ERR_UNSUPPORTED when the
 * layout cannot hold info's code.  The output is the same for every layout. */
int ecf8_bf16_decode_layout(const ecf8_bf16_info* info, const void* d_blob, const void* d_table, uint16_t* d_out,
                            size_t n, int32_t* d_status, cudaStream_t stream, int layout);

#ifdef __cplusplus
}
#endif
#endif /* ECF8_H_ */
