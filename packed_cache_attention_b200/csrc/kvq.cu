// libkvq C ABI: argument validation, buffer-size queries, table upload and kernel launches.
// The declarations, with the passages each operation follows, are in include/kvq.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "calibrate.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "nf4.cuh"
#include "quantize.cuh"

using namespace kvq;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_upload_mu;
bool g_uploaded[kMaxDevices] = {};

kvq_status ensure_tables() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_upload_mu);
  if (g_uploaded[dev]) return KVQ_OK;
  const Tables& t = tables();
  DevTables d;
  std::memcpy(d.centroid_f16, t.centroid_f16, sizeof(d.centroid_f16));
  std::memcpy(d.threshold, t.threshold, sizeof(d.threshold));
  std::memcpy(d.delta, t.delta, sizeof(d.delta));
  std::memcpy(d.nf4, t.nf4, sizeof(d.nf4));
  std::memcpy(d.nf4_mid, t.nf4_mid, sizeof(d.nf4_mid));
  if (cudaMemcpyToSymbol(c_tab, &d, sizeof(d)) != cudaSuccess) return KVQ_ERR_CUDA;
  static uint8_t lut[kLutBytes];
  decode_lut_image(t.centroid_f16, lut);
  if (cudaMemcpyToSymbol(g_dec_lut, lut, sizeof(lut)) != cudaSuccess) return KVQ_ERR_CUDA;
  static uint32_t qlut[2 * kLutEntries];
  if (!quant_lut_image(t.threshold, qlut)) return KVQ_ERR_UNSUPPORTED;
  if (cudaMemcpyToSymbol(g_quant_lut, qlut, sizeof(qlut)) != cudaSuccess) return KVQ_ERR_CUDA;
  g_uploaded[dev] = true;
  return KVQ_OK;
}

size_t elem_size(int dtype) {
  switch (dtype) {
    case KVQ_F32: return 4;
    case KVQ_F16: return 2;
    case KVQ_BF16: return 2;
    default: return 0;
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Checks a [B][H][T][128] view: supported dtype, positive sizes, 16-byte aligned rows.
kvq_status check_tensor(const void* ptr, const kvq_tensor4* t) {
  if (!ptr || !t) return KVQ_ERR_ARG;
  const size_t es = elem_size(t->dtype);
  if (es == 0) return KVQ_ERR_DTYPE;
  if (t->head_dim != kD) return KVQ_ERR_SHAPE;
  if (t->batch < 1 || t->n_heads < 1 || t->seq_len < 1) return KVQ_ERR_SHAPE;
  if (t->stride_b < 0 || t->stride_h < 0 || t->stride_t < 0) return KVQ_ERR_ARG;
  if (!aligned16(ptr)) return KVQ_ERR_ARG;
  if (((t->stride_b * es) % 16) || ((t->stride_h * es) % 16) || ((t->stride_t * es) % 16)) return KVQ_ERR_ARG;
  if (t->seq_len > 1 && t->stride_t < kD) return KVQ_ERR_ARG;
  return KVQ_OK;
}

bool cache_ok(const kvq_cache_desc* c) {
  return c && c->batch >= 1 && c->n_kv_heads >= 1 && c->head_dim == kD && c->capacity >= 1 && c->bits_k >= 1 &&
         c->bits_k <= 8 && c->bits_v >= 1 && c->bits_v <= 8;
}

size_t tile_record_bytes(int bits_k, int bits_v) { return 4ull * kD * (bits_k + bits_v) + 4ull * kTile; }

int n_tiles_of(int tokens) { return (tokens + kTile - 1) / kTile; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// NF4 decode: about 8 waves of two 16-warp CTAs per SM, so the hardware's CTA scheduling
// evens out the last wave, and at least one 32-token group per warp in every CTA.
int nf4_splits(int bh, int n_groups) {
  const int want = (16 * kTargetCtas + bh - 1) / bh;
  return std::max(1, std::min(std::min(want, n_groups / kNf4DecWarps), kMaxMergeSplits));
}

int decode_splits(int bh, int n_tiles) {
  const int want = (kTargetCtas + bh - 1) / bh;
  return std::max(1, std::min(std::min(want, n_tiles), kMaxMergeSplits));
}

// Block-GTQ decode: splits of whole 128-token chunks, about one CTA per SM in total.
int gtq_splits(int bh, int n_tiles) {
  const int n_chunks = (n_tiles + kChunkTiles - 1) / kChunkTiles;
  const int want = (kTargetCtas + bh - 1) / bh;
  return std::max(1, std::min(std::min(want, n_chunks), kMaxMergeSplits));
}

struct DecodeWs {
  size_t tickets, part_m, part_l, part_o, total;
};

// Workspace of the decode kernels: tickets (per row: one final counter, then one counter per
// merge group), then (m, l, O) partials for `entries` entries per row.
DecodeWs decode_ws_layout(int bh, int entries, int rows, int groups) {
  DecodeWs w;
  w.tickets = sizeof(WsHeader);
  w.part_m = align_up(w.tickets + 4ull * bh * (1 + groups), 128);
  w.part_l = align_up(w.part_m + 4ull * bh * entries * rows, 128);
  w.part_o = align_up(w.part_l + 4ull * bh * entries * rows, 128);
  w.total = align_up(w.part_o + 4ull * bh * entries * rows * kD, 128);
  return w;
}

int merge_groups(int splits) { return (splits + kMergeGroup - 1) / kMergeGroup; }

DecodeWs gtq_ws_layout(int bh, int splits) {
  const int groups = merge_groups(splits);
  return decode_ws_layout(bh, splits + groups, 8, groups);
}

int sm_count() {
  static int cached[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 148;
  }
  return cached[dev];
}

kvq_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

Nf4Layout nf4_layout(int batch, int n_heads, int capacity) {
  Nf4Layout L;
  L.nblk = n_heads * kD / KVQ_NF4_BLOCK;
  L.t_pad = (capacity + KVQ_NF4_PAD - 1) / KVQ_NF4_PAD * KVQ_NF4_PAD;
  L.codes_bytes = static_cast<size_t>(batch) * L.nblk * L.t_pad * 128;
  return L;
}

constexpr size_t kMaxSmem = 227 * 1024;

// Deepest bulk-copy pipeline (1..4 stages of 4 tile halves) that fits in shared memory.
int decode_stages(int bits_k, int bits_v) {
  const size_t per = static_cast<size_t>(kChunkTiles) * stage_tile_stride(bits_k, bits_v);
  const size_t room = kMaxSmem - decode_stage_off();
  return static_cast<int>(std::max<size_t>(1, std::min<size_t>(kDecStagesMax, room / per)));
}

size_t decode_smem_bytes(int bits_k, int bits_v) {
  const size_t stage =
      static_cast<size_t>(kChunkTiles) * stage_tile_stride(bits_k, bits_v) * decode_stages(bits_k, bits_v);
  // the stage area also holds the merge scratch (4 KB)
  return decode_stage_off() + std::max<size_t>(stage, 256 * sizeof(float4));
}

}  // namespace

extern "C" {

int kvq_abi_version(void) { return KVQ_ABI_VERSION; }

const char* kvq_status_string(int s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_ARG: return "invalid argument";
    case KVQ_ERR_SHAPE: return "unsupported shape";
    case KVQ_ERR_DTYPE: return "unsupported dtype";
    case KVQ_ERR_BUDGET: return "bit budget out of range";
    case KVQ_ERR_RANGE: return "sequence length out of range";
    case KVQ_ERR_WORKSPACE: return "workspace missing or too small";
    case KVQ_ERR_CUDA: return "CUDA error";
    case KVQ_ERR_TIMEOUT: return "device wait timed out";
    case KVQ_ERR_UNSUPPORTED: return "unsupported configuration";
    default: return "unknown status";
  }
}

kvq_status kvq_codebook(int width, uint16_t* centroids_f16, float* thresholds, float* delta) {
  if (width < 1 || width > 8) return KVQ_ERR_ARG;
  const Tables& t = tables();
  const int n = 1 << width;
  if (centroids_f16) std::memcpy(centroids_f16, t.centroid_f16 + centroid_offset(width), n * sizeof(uint16_t));
  if (thresholds) std::memcpy(thresholds, t.threshold + threshold_offset(width), (n - 1) * sizeof(float));
  if (delta) *delta = t.delta[width];
  return KVQ_OK;
}

kvq_status kvq_nf4_table(float* levels, float* midpoints) {
  const Tables& t = tables();
  if (levels) std::memcpy(levels, t.nf4, sizeof(t.nf4));
  if (midpoints) std::memcpy(midpoints, t.nf4_mid, sizeof(t.nf4_mid));
  return KVQ_OK;
}

size_t kvq_alloc_bytes(int n_kv_heads) {
  return n_kv_heads > 0 ? static_cast<size_t>(n_kv_heads) * sizeof(kvq_head_alloc) : 0;
}

}  // extern "C"
namespace {
struct CalibWsLayout {
  size_t head_count, seg_count, energy, seg_sum, chunk_sum, total;
  int n_chunks, n_seg;
};

CalibWsLayout calib_ws_layout(int batch, int n_kv_heads, int n_calib_tokens) {
  CalibWsLayout L;
  const long long N = static_cast<long long>(batch) * n_calib_tokens;
  L.n_chunks = static_cast<int>((N + kCalibChunk - 1) / kCalibChunk);
  L.n_seg = (L.n_chunks + kCalibSegment - 1) / kCalibSegment;
  L.head_count = sizeof(WsHeader);
  L.seg_count = align_up(L.head_count + 4ull * n_kv_heads, 128);
  L.energy = align_up(L.seg_count + 4ull * n_kv_heads * L.n_seg, 128);
  L.seg_sum = align_up(L.energy + 8ull * n_kv_heads * kH, 128);
  L.chunk_sum = align_up(L.seg_sum + 8ull * n_kv_heads * L.n_seg * kH, 128);
  L.total = align_up(L.chunk_sum + 8ull * n_kv_heads * L.n_chunks * kH, 128);
  return L;
}
}  // namespace
extern "C" {

size_t kvq_calibrate_workspace_bytes(int batch, int n_kv_heads, int n_calib_tokens) {
  if (batch < 1 || n_kv_heads < 1 || n_calib_tokens < 1) return 0;
  if (static_cast<long long>(batch) * n_calib_tokens > 0x7fffffffLL) return 0;
  return calib_ws_layout(batch, n_kv_heads, n_calib_tokens).total;
}

size_t kvq_packed_bytes(const kvq_cache_desc* c) {
  if (!cache_ok(c)) return 0;
  return static_cast<size_t>(c->batch) * c->n_kv_heads * n_tiles_of(c->capacity) * tile_record_bytes(c->bits_k, c->bits_v);
}

size_t kvq_decode_workspace_bytes(const kvq_cache_desc* c, int n_q_heads) {
  if (!cache_ok(c) || n_q_heads < 1) return 0;
  const int bh = c->batch * c->n_kv_heads;
  return gtq_ws_layout(bh, gtq_splits(bh, n_tiles_of(c->capacity))).total;
}

kvq_status kvq_init(void) { return ensure_tables(); }

kvq_status kvq_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < sizeof(WsHeader)) return KVQ_ERR_WORKSPACE;
  return cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)) == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

kvq_status kvq_workspace_status(const void* ws, void* stream, int* device_code) {
  if (!ws) return KVQ_ERR_WORKSPACE;
  unsigned int code = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&code, ws, sizeof(code), cudaMemcpyDeviceToHost, s) != cudaSuccess) return KVQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return KVQ_ERR_CUDA;
  if (device_code) *device_code = static_cast<int>(code);
  return code == 0 ? KVQ_OK : static_cast<kvq_status>(code);
}

kvq_status kvq_calibrate(const void* K, const kvq_tensor4* kd, const kvq_calib_params* p, void* alloc_out,
                         void* ws, size_t ws_bytes, void* stream) {
  kvq_status st = check_tensor(K, kd);
  if (st != KVQ_OK) return st;
  if (!p || !alloc_out) return KVQ_ERR_ARG;
  if (p->w_max < 1 || p->w_max > 8 || p->bits_k < 1 || p->bits_k > p->w_max) return KVQ_ERR_BUDGET;
  if (p->mode != KVQ_MODE_BLOCKGTQ && p->mode != KVQ_MODE_UNIFORM) return KVQ_ERR_ARG;
  if (p->n_calib < 0 || p->n_calib > kd->seq_len) return KVQ_ERR_RANGE;
  const int n_calib = p->n_calib == 0 ? kd->seq_len : p->n_calib;
  const size_t need = kvq_calibrate_workspace_bytes(kd->batch, kd->n_heads, n_calib);
  if (!ws || ws_bytes < need || !aligned16(ws)) return KVQ_ERR_WORKSPACE;
  if ((st = ensure_tables()) != KVQ_OK) return st;
  const long long N = static_cast<long long>(kd->batch) * n_calib;
  if (N > 0x7fffffffLL) return KVQ_ERR_RANGE;
  const CalibWsLayout L = calib_ws_layout(kd->batch, kd->n_heads, n_calib);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  CalibWs cws;
  cws.head_count = reinterpret_cast<unsigned*>(w8 + L.head_count);
  cws.seg_count = reinterpret_cast<unsigned*>(w8 + L.seg_count);
  cws.energy = reinterpret_cast<double*>(w8 + L.energy);
  cws.seg_sum = reinterpret_cast<double*>(w8 + L.seg_sum);
  cws.chunk_sum = reinterpret_cast<double*>(w8 + L.chunk_sum);
  const int n_chunks = L.n_chunks;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  dim3 grid((n_chunks + kCalibChunksPerCta - 1) / kCalibChunksPerCta, kd->n_heads);
  const int threads = 16 * kCalibChunksPerCta;
  switch (kd->dtype) {
    case KVQ_F32:
      kvq_calib_reduce<KVQ_F32><<<grid, threads, 0, s>>>(static_cast<const float*>(K), n_calib, kd->stride_b,
                                                         kd->stride_h, kd->stride_t, static_cast<int>(N), n_chunks, cws);
      break;
    case KVQ_F16:
      kvq_calib_reduce<KVQ_F16><<<grid, threads, 0, s>>>(static_cast<const __half*>(K), n_calib, kd->stride_b,
                                                         kd->stride_h, kd->stride_t, static_cast<int>(N), n_chunks, cws);
      break;
    default:
      kvq_calib_reduce<KVQ_BF16><<<grid, threads, 0, s>>>(static_cast<const __nv_bfloat16*>(K), n_calib, kd->stride_b,
                                                          kd->stride_h, kd->stride_t, static_cast<int>(N), n_chunks, cws);
  }
  if ((st = launch_status()) != KVQ_OK) return st;
  kvq_greedy_alloc<<<kd->n_heads, 512, 0, s>>>(cws.energy, p->bits_k, p->w_max, p->mode,
                                               static_cast<kvq_head_alloc*>(alloc_out));
  return launch_status();
}

namespace {

// Quantizes tokens t_begin .. t_begin + kd->seq_len - 1 (input row i = token t_begin + i) into
// their tiles of `packed`; the rest of a partly covered first tile keeps its stored codes.
kvq_status launch_quant(const void* K, const kvq_tensor4* kd, const void* V, const kvq_tensor4* vd, const void* alloc,
                        const kvq_cache_desc* c, int t_begin, void* packed, void* stream) {
  kvq_status st;
  if ((st = check_tensor(K, kd)) != KVQ_OK) return st;
  if ((st = check_tensor(V, vd)) != KVQ_OK) return st;
  if (!alloc || !packed || !aligned16(packed)) return KVQ_ERR_ARG;
  if (!cache_ok(c)) return KVQ_ERR_ARG;
  if (vd->dtype != kd->dtype || vd->batch != kd->batch || vd->n_heads != kd->n_heads || vd->seq_len != kd->seq_len)
    return KVQ_ERR_SHAPE;
  if (kd->batch != c->batch || kd->n_heads != c->n_kv_heads) return KVQ_ERR_SHAPE;
  if (t_begin < 0 || static_cast<long long>(t_begin) + kd->seq_len > c->capacity) return KVQ_ERR_RANGE;
  if ((st = ensure_tables()) != KVQ_OK) return st;
  const int t_end = t_begin + kd->seq_len;
  const int tile_lo = t_begin / kTile;
  const int n_tiles = n_tiles_of(t_end) - tile_lo;
  const int tiles_cap = n_tiles_of(c->capacity);
  const long long n_tasks = static_cast<long long>(c->batch) * c->n_kv_heads * n_tiles;
  if (n_tasks > 0x7fffffffLL - 4096LL * 64) return KVQ_ERR_RANGE;   // task indices are 32-bit
  const int rec = static_cast<int>(tile_record_bytes(c->bits_k, c->bits_v));
  const size_t smem = quant_smem_bytes(kd->dtype);
  const int qw = quant_warps(kd->dtype);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Persistent grid: exactly the CTAs that are resident at once (registers and shared memory
  // both limit it), so every warp starts at launch and the tiles are spread evenly.
  // The shared-memory opt-in and the occupancy query are made once per device, dtype and value
  // width (they cost host time comparable to a small launch, e.g. a one-token append).
  static std::mutex occ_mu;
  static int occ[kMaxDevices][24] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
#define KVQ_LAUNCH_QUANT(DT, TY, BV)                                                                              \
  do {                                                                                                            \
    auto kern = kvq_quant_pack<DT, BV>;                                                                           \
    int per_sm = 0;                                                                                               \
    {                                                                                                             \
      std::lock_guard<std::mutex> lock(occ_mu);                                                                   \
      if (occ[dev][DT * 8 + BV - 1] == 0) {                                                                       \
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=    \
            cudaSuccess)                                                                                          \
          return KVQ_ERR_CUDA;                                                                                    \
        int n = 0;                                                                                                \
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, qw * 32, smem) != cudaSuccess)                \
          return KVQ_ERR_CUDA;                                                                                    \
        occ[dev][DT * 8 + BV - 1] = std::max(1, n);                                                               \
      }                                                                                                           \
      per_sm = occ[dev][DT * 8 + BV - 1];                                                                         \
    }                                                                                                             \
    const long long want = (n_tasks + qw - 1) / qw;                                                             \
    const unsigned grid =                                                                                         \
        static_cast<unsigned>(std::min<long long>(want, static_cast<long long>(sm_count()) * std::max(1, per_sm))); \
    kern<<<grid, qw * 32, smem, s>>>(static_cast<const TY*>(K), kd->stride_b, kd->stride_h, kd->stride_t,         \
                                     static_cast<const TY*>(V), vd->stride_b, vd->stride_h, vd->stride_t, t_begin, \
                                     t_end, tile_lo, n_tiles, c->n_kv_heads, tiles_cap,                           \
                                     static_cast<const kvq_head_alloc*>(alloc), c->bits_k, c->bits_v,             \
                                     static_cast<uint8_t*>(packed), rec, static_cast<int>(n_tasks));              \
  } while (0)
#define KVQ_QUANT_BV(DT, TY)                                                                                      \
  switch (c->bits_v) {                                                                                            \
    case 1: KVQ_LAUNCH_QUANT(DT, TY, 1); break;                                                                   \
    case 2: KVQ_LAUNCH_QUANT(DT, TY, 2); break;                                                                   \
    case 3: KVQ_LAUNCH_QUANT(DT, TY, 3); break;                                                                   \
    case 4: KVQ_LAUNCH_QUANT(DT, TY, 4); break;                                                                   \
    case 5: KVQ_LAUNCH_QUANT(DT, TY, 5); break;                                                                   \
    case 6: KVQ_LAUNCH_QUANT(DT, TY, 6); break;                                                                   \
    case 7: KVQ_LAUNCH_QUANT(DT, TY, 7); break;                                                                   \
    default: KVQ_LAUNCH_QUANT(DT, TY, 8); break;                                                                  \
  }
  switch (kd->dtype) {
    case KVQ_F32: KVQ_QUANT_BV(KVQ_F32, float); break;
    case KVQ_F16: KVQ_QUANT_BV(KVQ_F16, __half); break;
    default: KVQ_QUANT_BV(KVQ_BF16, __nv_bfloat16); break;
  }
#undef KVQ_QUANT_BV
#undef KVQ_LAUNCH_QUANT
  return launch_status();
}

}  // namespace

kvq_status kvq_quantize(const void* K, const kvq_tensor4* kd, const void* V, const kvq_tensor4* vd, const void* alloc,
                        const kvq_cache_desc* c, void* packed, void* stream) {
  return launch_quant(K, kd, V, vd, alloc, c, 0, packed, stream);
}

kvq_status kvq_append(const void* K, const kvq_tensor4* kd, const void* V, const kvq_tensor4* vd, const void* alloc,
                      const kvq_cache_desc* c, int t_begin, void* packed, void* stream) {
  return launch_quant(K, kd, V, vd, alloc, c, t_begin, packed, stream);
}

kvq_status kvq_decode_attn(const void* q, const kvq_tensor4* qd, const void* packed, const void* alloc,
                           const kvq_cache_desc* c, int seq_len, float* out, void* ws, size_t ws_bytes,
                           void* stream) {
  kvq_status st;
  if ((st = check_tensor(q, qd)) != KVQ_OK) return st;
  if (!packed || !alloc || !out || !aligned16(packed) || !aligned16(alloc)) return KVQ_ERR_ARG;
  if (!cache_ok(c)) return KVQ_ERR_ARG;
  if (qd->seq_len != 1 || qd->batch != c->batch) return KVQ_ERR_SHAPE;
  if (qd->n_heads % c->n_kv_heads != 0 || qd->n_heads / c->n_kv_heads > 8) return KVQ_ERR_UNSUPPORTED;
  if (seq_len < 1 || seq_len > c->capacity) return KVQ_ERR_RANGE;
  const int bh = c->batch * c->n_kv_heads;
  const int n_tiles = n_tiles_of(seq_len);
  const int splits = gtq_splits(bh, n_tiles);
  const DecodeWs L = gtq_ws_layout(bh, splits);
  if (!ws || ws_bytes < L.total || !aligned16(ws) || ws_bytes < kvq_decode_workspace_bytes(c, qd->n_heads))
    return KVQ_ERR_WORKSPACE;
  if ((st = ensure_tables()) != KVQ_OK) return st;
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  const int rec = static_cast<int>(tile_record_bytes(c->bits_k, c->bits_v));
  const size_t smem = decode_smem_bytes(c->bits_k, c->bits_v);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  dim3 grid(splits, bh);
#define KVQ_LAUNCH_DEC(DT, TY, BV)                                                                                    \
  do {                                                                                                                \
    auto kern = kvq_decode_gtq<DT, BV>;                                                                               \
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=            \
        cudaSuccess)                                                                                                  \
      return KVQ_ERR_CUDA;                                                                                            \
    kern<<<grid, kDecThreads, smem, s>>>(                                                                             \
        static_cast<const TY*>(q), qd->stride_b, qd->stride_h, qd->n_heads, c->n_kv_heads,                             \
        static_cast<const uint8_t*>(packed), static_cast<const kvq_head_alloc*>(alloc), n_tiles_of(c->capacity), rec, \
        c->bits_k, c->bits_v, seq_len, splits, merge_groups(splits), decode_stages(c->bits_k, c->bits_v), out,       \
        reinterpret_cast<float*>(w8 + L.part_m), reinterpret_cast<float*>(w8 + L.part_l),                            \
        reinterpret_cast<float*>(w8 + L.part_o), reinterpret_cast<unsigned*>(w8 + L.tickets),                        \
        reinterpret_cast<unsigned*>(w8));                                                                             \
  } while (0)
#define KVQ_DEC_BV(DT, TY)                                                                                            \
  switch (c->bits_v) {                                                                                                \
    case 1: KVQ_LAUNCH_DEC(DT, TY, 1); break;                                                                         \
    case 2: KVQ_LAUNCH_DEC(DT, TY, 2); break;                                                                         \
    case 3: KVQ_LAUNCH_DEC(DT, TY, 3); break;                                                                         \
    case 4: KVQ_LAUNCH_DEC(DT, TY, 4); break;                                                                         \
    case 5: KVQ_LAUNCH_DEC(DT, TY, 5); break;                                                                         \
    case 6: KVQ_LAUNCH_DEC(DT, TY, 6); break;                                                                         \
    case 7: KVQ_LAUNCH_DEC(DT, TY, 7); break;                                                                         \
    default: KVQ_LAUNCH_DEC(DT, TY, 8); break;                                                                        \
  }
  switch (qd->dtype) {
    case KVQ_F32: KVQ_DEC_BV(KVQ_F32, float); break;
    case KVQ_F16: KVQ_DEC_BV(KVQ_F16, __half); break;
    default: KVQ_DEC_BV(KVQ_BF16, __nv_bfloat16); break;
  }
#undef KVQ_DEC_BV
#undef KVQ_LAUNCH_DEC
  return launch_status();
}

size_t kvq_nf4_packed_bytes(int batch, int n_heads, int capacity, int head_dim) {
  if (batch < 1 || n_heads < 2 || (n_heads & 1) || capacity < 1 || head_dim != kD) return 0;
  const Nf4Layout L = nf4_layout(batch, n_heads, capacity);
  return 2 * L.codes_bytes + 2 * (L.codes_bytes / 128) * sizeof(__half);
}

size_t kvq_nf4_decode_workspace_bytes(int batch, int n_heads, int capacity, int head_dim) {
  if (batch < 1 || n_heads < 1 || capacity < 1 || head_dim != kD) return 0;
  const int bh = batch * n_heads;
  return decode_ws_layout(bh, nf4_splits(bh, (capacity + 31) / 32), 1, 0).total;
}

namespace {

// NF4 rows t_begin .. t_begin + kd->seq_len - 1 of a cache of `capacity` tokens; padding rows
// after them are written up to t_stop.
kvq_status launch_nf4_quant(const void* K, const kvq_tensor4* kd, const void* V, const kvq_tensor4* vd,
                            int capacity, int t_begin, bool pad_to_capacity, void* packed, void* stream) {
  kvq_status st;
  if ((st = check_tensor(K, kd)) != KVQ_OK) return st;
  if ((st = check_tensor(V, vd)) != KVQ_OK) return st;
  if (!packed || !aligned16(packed)) return KVQ_ERR_ARG;
  if (vd->dtype != kd->dtype || vd->batch != kd->batch || vd->n_heads != kd->n_heads || vd->seq_len != kd->seq_len)
    return KVQ_ERR_SHAPE;
  if (kd->n_heads & 1) return KVQ_ERR_SHAPE;
  if (t_begin < 0 || static_cast<long long>(t_begin) + kd->seq_len > capacity) return KVQ_ERR_RANGE;
  if ((st = ensure_tables()) != KVQ_OK) return st;
  const Nf4Layout L = nf4_layout(kd->batch, kd->n_heads, capacity);
  const int t_end = t_begin + kd->seq_len;
  const int t_stop = pad_to_capacity ? L.t_pad
                                     : std::min(L.t_pad, (t_end + KVQ_NF4_PAD - 1) / KVQ_NF4_PAD * KVQ_NF4_PAD);
  const int groups = (t_stop + kNf4Rows - 1) / kNf4Rows - t_begin / kNf4Rows;
  const long long tasks = 2LL * kd->batch * L.nblk * groups;
  const unsigned grid = static_cast<unsigned>((tasks + kNf4Warps - 1) / kNf4Warps);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (kd->dtype) {
    case KVQ_F32:
      (pad_to_capacity ? kvq_nf4_quant_pack<KVQ_F32, false>
                       : kvq_nf4_quant_pack<KVQ_F32, true>)<<<grid, kNf4Warps * 32, 0, s>>>(
          static_cast<const float*>(K), kd->stride_b, kd->stride_h, kd->stride_t, static_cast<const float*>(V),
          vd->stride_b, vd->stride_h, vd->stride_t, kd->batch, t_begin, t_end, t_stop, L,
          static_cast<uint8_t*>(packed));
      break;
    case KVQ_F16:
      (pad_to_capacity ? kvq_nf4_quant_pack<KVQ_F16, false>
                       : kvq_nf4_quant_pack<KVQ_F16, true>)<<<grid, kNf4Warps * 32, 0, s>>>(
          static_cast<const __half*>(K), kd->stride_b, kd->stride_h, kd->stride_t, static_cast<const __half*>(V),
          vd->stride_b, vd->stride_h, vd->stride_t, kd->batch, t_begin, t_end, t_stop, L,
          static_cast<uint8_t*>(packed));
      break;
    default:
      (pad_to_capacity ? kvq_nf4_quant_pack<KVQ_BF16, false>
                       : kvq_nf4_quant_pack<KVQ_BF16, true>)<<<grid, kNf4Warps * 32, 0, s>>>(
          static_cast<const __nv_bfloat16*>(K), kd->stride_b, kd->stride_h, kd->stride_t,
          static_cast<const __nv_bfloat16*>(V), vd->stride_b, vd->stride_h, vd->stride_t, kd->batch, t_begin, t_end,
          t_stop, L, static_cast<uint8_t*>(packed));
  }
  return launch_status();
}

}  // namespace

kvq_status kvq_nf4_quantize(const void* K, const kvq_tensor4* kd, const void* V, const kvq_tensor4* vd, int capacity,
                            void* packed, void* stream) {
  return launch_nf4_quant(K, kd, V, vd, capacity, 0, true, packed, stream);
}

kvq_status kvq_nf4_append(const void* K, const kvq_tensor4* kd, const void* V, const kvq_tensor4* vd, int capacity,
                          int t_begin, void* packed, void* stream) {
  return launch_nf4_quant(K, kd, V, vd, capacity, t_begin, false, packed, stream);
}

kvq_status kvq_nf4_decode_attn(const void* q, const kvq_tensor4* qd, const void* packed, int capacity, int seq_len,
                               float* out, void* ws, size_t ws_bytes, void* stream) {
  kvq_status st;
  if ((st = check_tensor(q, qd)) != KVQ_OK) return st;
  if (!packed || !out) return KVQ_ERR_ARG;
  if (qd->seq_len != 1 || (qd->n_heads & 1)) return KVQ_ERR_SHAPE;
  if (seq_len < 1 || seq_len > capacity) return KVQ_ERR_RANGE;
  const int bh = qd->batch * qd->n_heads;
  const int splits = nf4_splits(bh, (seq_len + 31) / 32);
  const DecodeWs Lw = decode_ws_layout(bh, splits, 1, 0);
  if (!ws || ws_bytes < Lw.total || !aligned16(ws) ||
      ws_bytes < kvq_nf4_decode_workspace_bytes(qd->batch, qd->n_heads, capacity, kD))
    return KVQ_ERR_WORKSPACE;
  if ((st = ensure_tables()) != KVQ_OK) return st;
  const Nf4Layout L = nf4_layout(qd->batch, qd->n_heads, capacity);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  dim3 grid(splits, bh);
#define KVQ_LAUNCH_NF4DEC(DT, TY)                                                                              \
  kvq_nf4_decode<DT><<<grid, kNf4DecWarps * 32, 0, s>>>(                                                          \
      static_cast<const TY*>(q), qd->stride_b, qd->stride_h, qd->n_heads, static_cast<const uint8_t*>(packed), L, \
      seq_len, splits, out, reinterpret_cast<float*>(w8 + Lw.part_m), reinterpret_cast<float*>(w8 + Lw.part_l),  \
      reinterpret_cast<float*>(w8 + Lw.part_o), reinterpret_cast<unsigned*>(w8 + Lw.tickets))
  switch (qd->dtype) {
    case KVQ_F32: KVQ_LAUNCH_NF4DEC(KVQ_F32, float); break;
    case KVQ_F16: KVQ_LAUNCH_NF4DEC(KVQ_F16, __half); break;
    default: KVQ_LAUNCH_NF4DEC(KVQ_BF16, __nv_bfloat16); break;
  }
#undef KVQ_LAUNCH_NF4DEC
  return launch_status();
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// Decode attention for callers that cannot allocate device memory.
//
// Some hosts of this library hand it only their input and output buffers and own no device
// allocator of their own: a plain-C host that never links a CUDA memory manager, or an
// inference-engine plugin whose interface forbids allocating on the hot path. They cannot
// provide the split-merge workspace kvq_decode_attn needs. This entry point uses a fixed
// scratch array instead: a file-scope __device__ array that every GPU loading the library
// holds until the process exits. Its device address is looked up once per device (with that
// device current) and handed to the ordinary decode kernel as its workspace.
namespace {

constexpr size_t kNoAllocScratchBytes = 2u << 20;   // 2 MiB per device
__device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device. The first call on a device
// resolves it with cudaGetSymbolAddress and zeroes the array (the split tickets in it must
// start at zero; the kernel returns them to zero after every call).
kvq_status decode_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return KVQ_ERR_CUDA;
    if (cudaMemset(p, 0, kNoAllocScratchBytes) != cudaSuccess) return KVQ_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return KVQ_OK;
}

}  // namespace

extern "C" {

size_t kvq_decode_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

kvq_status kvq_decode_attn_noalloc(const void* q, const kvq_tensor4* qd, const void* packed, const void* alloc,
                                   const kvq_cache_desc* cache, int seq_len, float* out, void* stream) {
  if (!qd || !cache_ok(cache)) return KVQ_ERR_ARG;
  const size_t need = kvq_decode_workspace_bytes(cache, qd->n_heads);
  if (need == 0) return KVQ_ERR_ARG;
  if (need > kNoAllocScratchBytes) return KVQ_ERR_WORKSPACE;
  kvq_status st = ensure_tables();
  if (st != KVQ_OK) return st;
  void* scratch = nullptr;
  if ((st = decode_scratch(&scratch)) != KVQ_OK) return st;
  return kvq_decode_attn(q, qd, packed, alloc, cache, seq_len, out, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"

