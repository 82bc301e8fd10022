/*
 * libkvq — packed KV-cache quantization and fused decode attention for NVIDIA B200 (sm_100a).
 *
 * C ABI. Every data pointer is a DEVICE pointer unless the comment says "host". The caller
 * owns all memory; the library never allocates. Buffer sizes come from the kvq_*_bytes
 * queries. Every launch is asynchronous on the stream passed as `stream` (a cudaStream_t,
 * NULL = legacy default stream). Argument errors are detected on the host and returned
 * before anything is launched. A launch failure returns KVQ_ERR_CUDA. Device-side failures
 * (a bounded wait that ran out) are recorded in the workspace's status word and read back
 * with kvq_workspace_status(). No C++ exception crosses this boundary.
 *
 * The first call that launches work on a device uploads the constant tables (codebooks, NF4
 * levels) to that device with a synchronous copy, so it must not be made while a stream is
 * being captured; kvq_init() does the upload explicitly.
 *
 * Host threads may call the library at once: its one-time setup per device and CUDA context
 * (tables, kernel attributes, occupancy) is serialized inside it. Calls that share a workspace
 * or write the same packed cache must still not overlap on the GPU.
 *
 * Calibrate, quantize/append and the Block-GTQ decode are launched with programmatic
 * dependent launch: such a kernel may start (barriers, tensor memory, the library's own tables)
 * while the previous kernel in the stream is finishing, but reads and writes none of the
 * caller's memory until that kernel has completed, so stream order holds as for any launch.
 *
 * Sources (restated in each declaration):
 *   [BGTQ] "RoPE-aware bit allocation for KV cache quantization" (Liang, Zhang, Jia;
 *          arXiv 2606.24033), abstract.
 *   [NQKV] review of "NQKV: A KV Cache Quantization Scheme Based on Normal Distribution
 *          Characteristics" (arXiv 2505.16210): mechanism paragraph, referee major
 *          comment 1, assumptions, Figs. 5-7.
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVQ_ABI_VERSION 4
#define KVQ_TILE_TOKENS 32     /* tokens per packed Block-GTQ tile */
#define KVQ_HEAD_DIM 128       /* head dimension the kernels are built for */
#define KVQ_MAX_WIDTH 8        /* widest Lloyd-Max codebook */
#define KVQ_NF4_BLOCK 256      /* values per NF4 block */
#define KVQ_NF4_PAD 16         /* NF4 token padding multiple */

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_ARG = 1,          /* null pointer, bad stride or alignment, inconsistent sizes */
  KVQ_ERR_SHAPE = 2,        /* shape the kernels do not support (e.g. head_dim != 128) */
  KVQ_ERR_DTYPE = 3,        /* unknown element type */
  KVQ_ERR_BUDGET = 4,       /* bit budget outside 1..w_max or w_max outside 1..8 */
  KVQ_ERR_RANGE = 5,        /* seq_len beyond the buffer's capacity */
  KVQ_ERR_WORKSPACE = 6,    /* workspace missing or smaller than the size query says */
  KVQ_ERR_CUDA = 7,         /* a CUDA runtime call or launch failed */
  KVQ_ERR_TIMEOUT = 8,      /* a device-side bounded wait gave up (read via kvq_workspace_status) */
  KVQ_ERR_UNSUPPORTED = 9,  /* a combination the library does not implement */
  KVQ_ERR_MISMATCH = 10     /* packed cache header disagrees with the descriptor or the allocation */
} kvq_status;

typedef enum { KVQ_F32 = 0, KVQ_F16 = 1, KVQ_BF16 = 2 } kvq_dtype;

typedef enum { KVQ_MODE_BLOCKGTQ = 0, KVQ_MODE_UNIFORM = 1 } kvq_mode;

/* A [batch][n_heads][seq_len][head_dim] tensor view. Strides are in elements; the last
 * dimension is contiguous. Every row start must be 16-byte aligned. */
typedef struct {
  int32_t batch;
  int32_t n_heads;
  int32_t seq_len;
  int32_t head_dim;
  int64_t stride_b;
  int64_t stride_h;
  int64_t stride_t;
  int32_t dtype;            /* kvq_dtype */
  int32_t reserved;
} kvq_tensor4;

/* Calibration settings. bits_k: K budget in bits per dimension (1..w_max). w_max: widest
 * width a block may receive (1..8; 8 recommended). n_calib: leading tokens of every
 * sequence used for the energy score (0 = all). mode: kvq_mode. */
typedef struct {
  int32_t bits_k;
  int32_t w_max;
  int32_t n_calib;
  int32_t mode;
} kvq_calib_params;

/* Shape of one packed Block-GTQ cache buffer (one layer). capacity = tokens per sequence
 * the buffer holds; storage is rounded up to whole 32-token tiles. bits_v = 0 makes a
 * keys-only cache: the records hold no values, and the decode reads them from the caller's
 * unquantized value tensor (kvq_decode_attn_ex). */
typedef struct {
  int32_t batch;
  int32_t n_kv_heads;
  int32_t head_dim;
  int32_t capacity;
  int32_t bits_k;
  int32_t bits_v;
} kvq_cache_desc;

/* Allocation record of one KV head, as written by kvq_calibrate (device memory, array of
 * n_kv_heads records). Block b covers dims b and b + head_dim/2.
 * A token's K codes form one bit stream in "stream order": width classes from 8 bits down
 * to 1 bit, blocks ascending within a class, each block contributing the code of dim b and
 * then the code of dim b + head_dim/2; blocks of width 0 contribute nothing. */
typedef struct {
  double energy[64];        /* E_b, mean ||k_b||^2 over the calibration tokens */
  float gain[64];           /* g_b, per-block scale applied before the codebook */
  float dequant[64];        /* f_b = 1 / (sqrt(d) g_b) */
  int16_t bit_off[64];      /* bit offset of block b's code pair in the K stream (-1: width 0) */
  uint8_t width[64];        /* w_b, bits per dim of block b */
  uint8_t stream_block[64]; /* blocks in stream order; 255 after the last one */
  uint16_t class_bit[8];    /* class c (stream order): bit offset of its first code */
  uint8_t class_width[8];   /* class c: width (0 = no such class) */
  uint8_t class_first[8];   /* class c: index of its first block in stream_block */
  uint8_t class_blocks[8];  /* class c: number of blocks */
  uint8_t reserved_b[56];
  int32_t head_dim;
  int32_t bits_k;
  int32_t w_max;
  int32_t mode;
  int32_t n_classes;        /* number of classes with at least one block */
  int32_t k_words;          /* 32-bit words in a tile's K part (= bits_k * head_dim) */
  int32_t n_blocks;         /* blocks with w_b > 0 */
  int32_t reserved;
  /* Decode plan (written by kvq_calibrate, read by the decode). The K operand of the
   * tensor-core product has one column per block pair. Each width class, in stream order, is
   * cut into slots of 4 consecutive block pairs; a class's last slot holds the 1..4 pairs left
   * and the rest of it is padding. Slot s fills columns 4 s .. 4 s + 3. */
  uint32_t plan_slot[24];       /* width | bit offset of the slot's first pair in the K stream << 8 */
  int8_t plan_col_block[96];    /* block of column c, -1 for a padding column */
  int32_t plan_n_slots;
  int32_t plan_k_cols;          /* columns of the product: 4 * plan_n_slots rounded up to 8 */
  uint64_t digest;              /* sum mod 2^64 over blocks b of splitmix64(b << 40 | w_b << 32 |
                                   fp32 bits of g_b); also stored in the packed header */
  uint8_t reserved_c[432];
} kvq_head_alloc;

/* Header at offset 0 of every packed Block-GTQ cache (kvq_packed_header_bytes(n_kv_heads)
 * bytes; the tile records follow it). Written by kvq_quantize and by kvq_append with
 * t_begin = 0; checked by kvq_append (t_begin > 0) and by the decode, which refuse a cache
 * whose header disagrees with their descriptor or allocation (KVQ_ERR_MISMATCH) instead of
 * returning attention over misread codes. */
typedef struct {
  uint32_t magic;           /* 0x3151564B, the bytes "KVQ1" */
  uint16_t layout_version;  /* 1 */
  uint16_t head_dim;
  uint8_t bits_k;
  uint8_t bits_v;           /* 0: keys only */
  uint8_t w_max;
  uint8_t mode;
  uint32_t status;          /* 0, or the kvq_status of an append that found a mismatch */
  int32_t batch;
  int32_t n_kv_heads;
  int32_t capacity;
  uint32_t record_bytes;    /* bytes of one 32-token tile record */
  uint8_t reserved[32];
  /* followed (at byte 64) by uint64_t digest[n_kv_heads] (each head's kvq_head_alloc.digest), then zero
   * padding to a multiple of 128 bytes */
} kvq_packed_header;

/* ---------------------------------------------------------------- queries (host only) */

int kvq_abi_version(void);
const char* kvq_status_string(int status);

/* Host copy of the width-w Lloyd-Max codebook (w = 1..8) for N(0,1), as used by the
 * kernels: 2^w centroids as fp16 bit patterns, 2^w - 1 fp32 thresholds (midpoints of
 * adjacent fp16 centroids) and delta = fp32 MSE of that quantizer on N(0,1).
 * Any output pointer (host) may be NULL. [BGTQ]: TQ-MSE is the base quantizer. */
kvq_status kvq_codebook(int width, uint16_t* centroids_f16, float* thresholds, float* delta);

/* Host copy of the 16 NF4 levels (fp32, ascending) and 15 fp32 midpoints.
 * [NQKV] mechanism paragraph: 16 standard-normal quantiles imported from QLoRA. */
kvq_status kvq_nf4_table(float* levels, float* midpoints);

/* Bytes of the allocation buffer for n_kv_heads heads (n_kv_heads * sizeof(kvq_head_alloc) = 2048 each). */
size_t kvq_alloc_bytes(int n_kv_heads);

/* Workspace bytes kvq_calibrate needs for this many sequences, KV heads and calibration
 * tokens per sequence. */
size_t kvq_calibrate_workspace_bytes(int batch, int n_kv_heads, int n_calib_tokens);

/* Bytes of the header that starts every packed cache: 64 + 8 * n_kv_heads, rounded up to a
 * multiple of 128 (0 for n_kv_heads < 1). */
size_t kvq_packed_header_bytes(int n_kv_heads);

/* Bytes of one packed cache: the header, then batch * n_kv_heads * ceil(capacity/32) tile
 * records of 4 * head_dim * (bits_k + bits_v) + 128 bytes (keys only, bits_v = 0:
 * 4 * head_dim * bits_k + 64 bytes). Returns 0 for an invalid descriptor. */
size_t kvq_packed_bytes(const kvq_cache_desc* cache);

/* Workspace bytes kvq_decode_attn needs for this cache and n_q_heads query heads (any
 * seq_len up to the capacity). */
size_t kvq_decode_workspace_bytes(const kvq_cache_desc* cache, int n_q_heads);

/* ---------------------------------------------------------------- setup and status */

/* Uploads the constant tables to the current device (synchronous). Optional: the first
 * launching call does it too. */
kvq_status kvq_init(void);

/* Zero a decode or calibrate workspace (async memset on `stream`). Both hold counters that
 * must start at zero: zero a workspace once before its first use; the kernels return the
 * counters to zero, so it stays reusable for every call on the same cache descriptor (the
 * decode's counters sit where the descriptor's capacity puts them, whatever seq_len). Zero
 * it again before using it with a descriptor of another batch, head count or capacity.
 * Calls sharing one workspace must not overlap. */
kvq_status kvq_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Synchronizes `stream`, copies the workspace status word to *device_code (host) and
 * returns KVQ_OK if it is 0, else the recorded kvq_status (e.g. KVQ_ERR_TIMEOUT,
 * KVQ_ERR_MISMATCH). */
kvq_status kvq_workspace_status(const void* ws, void* stream, int* device_code);

/* Synchronizes `stream` and copies the status word of a packed cache's header to
 * *device_code (host): 0, or KVQ_ERR_MISMATCH left by an append that refused to extend it.
 * Returns KVQ_OK if it is 0, else that status. */
kvq_status kvq_packed_status(const void* packed, void* stream, int* device_code);

/* Text of the CUDA error behind the last KVQ_ERR_CUDA this process got from the library
 * ("no error" if there was none). Host only. */
const char* kvq_last_cuda_error(void);

/* Test hook for the bounded waits of the Block-GTQ decode: later decode calls give up a wait
 * after wait_limit tries (about 1 ms each; default 2000), and with no_loads != 0 they issue
 * no copy at all, so their first wait on a stage runs out with no work in flight: the call
 * then records KVQ_ERR_TIMEOUT in its workspace and writes nothing. Process-wide; meant
 * for tests, never for production calls. Returns KVQ_ERR_ARG for wait_limit < 1. */
kvq_status kvq_debug_decode(int wait_limit, int no_loads);

/* ---------------------------------------------------------------- Block-GTQ hot path */

/* Calibration ([BGTQ] abstract: per layer and KV head, a label-free energy score for every
 * RoPE block, then a greedy integer bit allocation by marginal gain).
 * K: keys [batch][n_kv_heads][seq_len][128] in kd->dtype (post-RoPE, as cached).
 * Two launches: a fixed-order fp64 reduction of E_b = mean_t (k_b^2 + k_{b+64}^2) over the
 * first n_calib tokens of every sequence (pooled), then the greedy allocation:
 * bits_k * 64 steps, each adding one bit to the block with the largest
 * E_b (delta(w_b) - delta(w_b + 1)) below w_max, ties to the lowest block.
 * The sum runs in a fixed order (64-token chunks, 64-chunk segments, segments), so the
 * energies are reproducible bit for bit.
 * Writes n_kv_heads kvq_head_alloc records to alloc_out.
 * ws: workspace of kvq_calibrate_workspace_bytes(batch, n_kv_heads, n_calib) bytes, zeroed
 * once by kvq_workspace_init. */
kvq_status kvq_calibrate(const void* K, const kvq_tensor4* kd, const kvq_calib_params* params,
                         void* alloc_out, void* ws, size_t ws_bytes, void* stream);

/* Quantize and pack the first kd->seq_len tokens of K and V into `packed` ([BGTQ]: Block-GTQ
 * on TQ-MSE, matched K/V budgets, packed cache). Per token row: fp16 norm, a = sqrt(d)/norm,
 * y = (x a) g_b in fp32, code = number of thresholds below y; K uses the allocation's
 * widths and gains, V uses width cache->bits_v and g = 1. Writes the packed header (see
 * kvq_packed_header). Tiles past seq_len are not written; tokens of the last tile beyond
 * seq_len are stored as code 0, norm 0.
 * Layout after the header: per (sequence, KV head) consecutive 32-token tile records of
 * 4 * head_dim * (bits_k + bits_v) + 128 bytes, little-endian:
 *   K part: 32-bit word 32 i + t is word i (i < 4 bits_k) of token t's K stream (see
 *           kvq_head_alloc; codes least significant bit first, bits_k * head_dim bits).
 *   32 fp16 K norms, then 32 fp16 V norms, in token order.
 *   V part: word 128 i + j is word i (i < bits_v) of dim j's V stream: the codes of the
 *           tile's tokens 0..31 at dim j, bits_v bits each, least significant bit first.
 * A keys-only cache (cache->bits_v = 0) stores the K part and the K norms only (records of
 * 4 * head_dim * bits_k + 64 bytes); V and vd may then be NULL.
 * K, V: [batch][n_kv_heads][seq_len][128] (kd, vd may differ in strides, not in shape).
 * alloc: records from kvq_calibrate with bits_k == cache->bits_k.
 * packed: kvq_packed_bytes(cache) bytes, 16-byte aligned. */
kvq_status kvq_quantize(const void* K, const kvq_tensor4* kd, const void* V, const kvq_tensor4* vd,
                        const void* alloc, const kvq_cache_desc* cache, void* packed, void* stream);

/* Append tokens to a packed cache ([NQKV] assumptions: the cache only grows, so new tokens are
 * encoded without re-quantizing the stored ones; Fig. 6, decoding phase: each new token's
 * keys and values are quantized and appended). Quantizes tokens t_begin .. t_begin + n - 1,
 * n = kd->seq_len, exactly as kvq_quantize quantizes them (the per-row quantizer depends on
 * nothing but the row and the allocation), so appending a sequence in any number of calls
 * stores the same bytes as one kvq_quantize call.
 * K, V: [batch][n_kv_heads][n][128]; input row i is token t_begin + i. Codes and norms of
 * tokens below t_begin in the first touched tile are kept (read back and merged); tokens from
 * t_begin + n to the end of the last touched tile are stored as code 0, norm 0. Tiles before
 * t_begin / 32 and after the last touched tile are not accessed.
 * An append with t_begin = 0 writes the packed header. One with t_begin > 0 first checks it on
 * the device: if it does not name this descriptor's shapes and widths and this allocation
 * (or already holds a status), the call writes nothing and leaves KVQ_ERR_MISMATCH in the
 * header's status word (kvq_packed_status; the decode reports it too).
 * Requires 0 <= t_begin and t_begin + n <= cache->capacity (else KVQ_ERR_RANGE); the stored
 * tokens below t_begin must have been written by an earlier call on the same stream (or one
 * that has completed). Attend over the grown cache with kvq_decode_attn(seq_len = t_begin + n). */
kvq_status kvq_append(const void* K, const kvq_tensor4* kd, const void* V, const kvq_tensor4* vd,
                      const void* alloc, const kvq_cache_desc* cache, int t_begin, void* packed, void* stream);

/* Fused decode attention straight from the packed cache ([BGTQ]: packed-cache serving path).
 * q: [batch][n_q_heads][1][128] (qd->seq_len must be 1), query head hq reads KV head
 * hq / (n_q_heads / n_kv_heads); n_q_heads / n_kv_heads must be 1..8.
 * out: fp32 [batch][n_q_heads][128], contiguous. Attends over cached positions
 * 0..seq_len-1: out = sum_t softmax_t(q . k_hat_t / sqrt(d)) v_hat_t with
 * k_hat = norm * c[code] * f_b and v_hat = norm * c[code] / sqrt(d).
 * packed, alloc: 16-byte aligned (as allocated by any CUDA allocator).
 * ws: kvq_decode_workspace_bytes bytes, zeroed once by kvq_workspace_init.
 * The kernel checks the packed header against `cache` and `alloc` (per-head digest): on a
 * mismatch, or a status an append left in the header, it records KVQ_ERR_MISMATCH in the
 * workspace status word and writes nothing. Keys-only caches (bits_v = 0) need the values:
 * use kvq_decode_attn_ex (KVQ_ERR_UNSUPPORTED here). */
kvq_status kvq_decode_attn(const void* q, const kvq_tensor4* qd, const void* packed, const void* alloc,
                           const kvq_cache_desc* cache, int seq_len, float* out, void* ws,
                           size_t ws_bytes, void* stream);

/* Extra inputs of kvq_decode_attn_ex. Every pointer may be NULL (then its view is ignored).
 * V, vd: the values of a keys-only cache (cache->bits_v = 0; the Block-GTQ page reports key
 *   errors with only the keys quantized, values left as they are):
 *   [batch][n_kv_heads][>= seq_len][128] in bf16 or fp16, row t = value of cached position t. Required for a keys-only cache, not
 *   allowed with packed values.
 * K_recent, V_recent, krd, vrd: the n_recent = krd.seq_len most recent tokens kept
 *   unquantized (the Block-GTQ page reports its results with no buffer of fp16 recent keys,
 *   which names this variant; here both their keys and values stay in the caller's dtype):
 *   [batch][n_kv_heads][n_recent][128] each, any dtype; they are cached positions seq_len ..
 *   seq_len + n_recent - 1 and join the packed positions in one softmax. */
typedef struct {
  const void* V;
  kvq_tensor4 vd;
  const void* K_recent;
  kvq_tensor4 krd;
  const void* V_recent;
  kvq_tensor4 vrd;
} kvq_decode_extra;

/* kvq_decode_attn with the extra inputs above: out = sum over packed positions 0..seq_len-1
 * and recent positions of softmax(q . k / sqrt(d)) v, where packed positions use k_hat (and
 * v_hat, or the dense values of a keys-only cache) and recent positions their exact k and v.
 * seq_len may be 0 when n_recent >= 1. Same workspace, header checks and status as
 * kvq_decode_attn; extra = NULL is kvq_decode_attn. A keys-only cache above 4 bits per dim
 * returns KVQ_ERR_UNSUPPORTED (its chunk stages, 128 value rows each, do not fit in the
 * decode's shared memory). */
kvq_status kvq_decode_attn_ex(const void* q, const kvq_tensor4* qd, const void* packed, const void* alloc,
                              const kvq_cache_desc* cache, int seq_len, const kvq_decode_extra* extra, float* out,
                              void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- NQKV-style NF4 variant */

/* Bytes of an NF4 cache for K and V: per (sequence, 256-value block): T_pad rows of 128
 * code bytes, for K then V, followed by fp16 scales for K then V; T_pad = ceil(capacity/16)*16. */
size_t kvq_nf4_packed_bytes(int batch, int n_heads, int capacity, int head_dim);

/* Workspace bytes kvq_nf4_decode_attn needs. */
size_t kvq_nf4_decode_workspace_bytes(int batch, int n_heads, int capacity, int head_dim);

/* NF4 quantize ([NQKV]: blocks of 256 values along each token's head-major hidden vector,
 * scale = fp16(absmax) with no mean subtraction, index = nearest NF4 level, 2 nibbles per
 * byte with value 2k in the low nibble of byte k; token rows padded to a multiple of 16).
 * K, V: [batch][n_heads][seq_len][128], n_heads even. Rows seq_len..T_pad-1 are written as
 * code 0, scale 0. */
kvq_status kvq_nf4_quantize(const void* K, const kvq_tensor4* kd, const void* V, const kvq_tensor4* vd,
                            int capacity, void* packed, void* stream);

/* NF4 append ([NQKV] assumptions: the cache only grows, so a new token's blocks are encoded
 * without re-quantizing stored ones; Fig. 6, decoding phase). Quantizes tokens t_begin ..
 * t_begin + n - 1 (n = kd->seq_len; input row i is token t_begin + i) exactly as
 * kvq_nf4_quantize does, writes padding rows (code 0, scale 0) from t_begin + n up to the next
 * multiple of 16, and leaves every other row untouched. Requires 0 <= t_begin and
 * t_begin + n <= capacity (else KVQ_ERR_RANGE). Rows below the next multiple of 16 after the
 * last token then hold the same bytes as one kvq_nf4_quantize call over all tokens. */
kvq_status kvq_nf4_append(const void* K, const kvq_tensor4* kd, const void* V, const kvq_tensor4* vd,
                          int capacity, int t_begin, void* packed, void* stream);

/* NF4 MHA decode attention ([NQKV]: dequantization is a table lookup; padding zeros are
 * masked): out[b][h] = sum_t softmax_t(q . x_hat / sqrt(d)) v_hat over t < seq_len with
 * x_hat = scale * NF4[idx]. q: [batch][n_heads][1][128]; out fp32 [batch][n_heads][128]. */
kvq_status kvq_nf4_decode_attn(const void* q, const kvq_tensor4* qd, const void* packed, int capacity,
                               int seq_len, float* out, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- allocation-free decode */

/* Decode attention for callers that cannot allocate device memory. No counterpart on the
 * pages: it is a convenience of this library. Some hosts give the library only their
 * input and output buffers and have no device allocator of their own (a plain-C host that
 * links no CUDA memory manager, an engine plugin whose interface forbids allocating on the
 * hot path), so they cannot supply the workspace kvq_decode_attn takes. This call computes
 * exactly what kvq_decode_attn computes (same arguments, without ws / ws_bytes) and uses as
 * its workspace a fixed scratch array of kvq_decode_noalloc_scratch_bytes() bytes (2 MiB)
 * that the library holds in device memory on every GPU that loads it, until the process
 * exits. It calls no cudaMalloc, cudaFree or other allocating routine. It covers the
 * Block-GTQ decode only (the NF4 decode has no allocation-free form).
 * - The array's address is looked up on every call. The first call on a device (and the
 *   first after its context was created again) zeroes the array with an asynchronous memset
 *   on `stream`, ordered before the decode; make that first call before any stream capture.
 * - The array's first 64 KiB hold the status word and the split counters of every call, the
 *   partials follow. Shapes whose counters (batch * n_kv_heads rows) do not fit there, or
 *   whose partials do not fit in the rest, return KVQ_ERR_WORKSPACE before anything is
 *   launched.
 * - Every call on a device shares the one array, which keeps the last call's contents; the
 *   split counters, which must start at zero, are returned to zero by every call and never
 *   share bytes with partials, so calls on caches of different shapes can follow each
 *   other. Calls that overlap on the GPU (other streams, other host threads) race on it:
 *   serialize them.
 * - A device-side wait that gave up is recorded in the array's status word; read it with
 *   kvq_decode_noalloc_status. */
kvq_status kvq_decode_attn_noalloc(const void* q, const kvq_tensor4* qd, const void* packed, const void* alloc,
                                   const kvq_cache_desc* cache, int seq_len, float* out, void* stream);

/* Size in bytes of the scratch array kvq_decode_attn_noalloc uses (2 MiB). */
size_t kvq_decode_noalloc_scratch_bytes(void);

/* Status of the allocation-free decode on the current device: synchronizes `stream`, copies
 * the scratch array's status word to *device_code (host) and clears it. Returns KVQ_OK if it
 * was 0, else the recorded kvq_status (e.g. KVQ_ERR_TIMEOUT). */
kvq_status kvq_decode_noalloc_status(void* stream, int* device_code);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */
