// libkvq C ABI: argument validation, buffer-size queries, table upload and kernel launches.
// The declarations, with the passages each operation follows, are in include/kvq.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstddef>
#include <cstring>
#include <mutex>
#include <utility>

#include "calibrate.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "nf4.cuh"
#include "quantize.cuh"

using namespace kvq;

namespace {

constexpr int kMaxDevices = 64;

// Last CUDA error behind a KVQ_ERR_CUDA of this process (kvq_last_cuda_error).
std::atomic<int> g_last_cuda_error{0};

kvq_status cuda_fail(cudaError_t e) {
  g_last_cuda_error.store(static_cast<int>(e));
  return KVQ_ERR_CUDA;
}

// Identity of the calling thread's current CUDA context. Per-device state the library sets up
// once (uploaded tables, shared-memory opt-ins, occupancy) is keyed on it, so a device whose
// context was reset and created again gets that state again instead of trusting a stale flag.
// The two driver functions are reached through the runtime, so the library has no link-time
// dependency on the driver library. Returns 1 when the identity cannot be read (then every
// context of the device counts as one).
uint64_t context_id() {
  using GetCurrent = int (*)(void**);
  using GetId = int (*)(void*, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(f);
  });
  if (!get_current || !get_id) return 1;
  void* ctx = nullptr;
  if (get_current(&ctx) != 0) return 1;
  if (!ctx) {                               // no runtime call has made the primary context current yet
    cudaFree(nullptr);
    if (get_current(&ctx) != 0 || !ctx) return 1;
  }
  unsigned long long id = 0;
  if (get_id(ctx, &id) != 0) return 1;
  return static_cast<uint64_t>(id) + 2;
}

std::mutex g_upload_mu;
uint64_t g_uploaded[kMaxDevices] = {};      // context the tables were uploaded to (0: none)

kvq_status ensure_tables() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
  const uint64_t ctx = context_id();
  std::lock_guard<std::mutex> lock(g_upload_mu);
  if (g_uploaded[dev] == ctx) return KVQ_OK;
  const Tables& t = tables();
  DevTables d;
  std::memcpy(d.centroid_f16, t.centroid_f16, sizeof(d.centroid_f16));
  std::memcpy(d.threshold, t.threshold, sizeof(d.threshold));
  std::memcpy(d.delta, t.delta, sizeof(d.delta));
  std::memcpy(d.nf4, t.nf4, sizeof(d.nf4));
  std::memcpy(d.nf4_mid, t.nf4_mid, sizeof(d.nf4_mid));
  { const cudaError_t e_ = cudaMemcpyToSymbol(c_tab, &d, sizeof(d)); if (e_ != cudaSuccess) return cuda_fail(e_); }
  static uint8_t lut[kLutBytes];
  decode_lut_image(t.centroid_f16, lut);
  { const cudaError_t e_ = cudaMemcpyToSymbol(g_dec_lut, lut, sizeof(lut)); if (e_ != cudaSuccess) return cuda_fail(e_); }
  static uint32_t qlut[2 * kLutEntries];
  if (!quant_lut_image(t.threshold, qlut)) return KVQ_ERR_UNSUPPORTED;
  { const cudaError_t e_ = cudaMemcpyToSymbol(g_quant_lut, qlut, sizeof(qlut)); if (e_ != cudaSuccess) return cuda_fail(e_); }
  static uint32_t nlut[2 * kNf4LutCells];
  if (!nf4_lut_image(t.nf4_mid, nlut)) return KVQ_ERR_UNSUPPORTED;
  { const cudaError_t e_ = cudaMemcpyToSymbol(g_nf4_lut, nlut, sizeof(nlut)); if (e_ != cudaSuccess) return cuda_fail(e_); }
  g_uploaded[dev] = ctx;
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
         c->bits_k <= 8 && c->bits_v >= 0 && c->bits_v <= 8;
}

// Record of 32 tokens: K words, K norms, then (unless keys only) V norms and V words.
size_t tile_record_bytes(int bits_k, int bits_v) {
  return bits_v == 0 ? 4ull * kD * bits_k + 2ull * kTile : 4ull * kD * (bits_k + bits_v) + 4ull * kTile;
}

// Packed header: 64 bytes of fields and one 64-bit digest per KV head, padded to 128 bytes.
size_t header_bytes(int n_kv_heads) { return (64ull + 8ull * n_kv_heads + 127) / 128 * 128; }

int n_tiles_of(int tokens) { return (tokens + kTile - 1) / kTile; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int sm_count();

// NF4 decode: about 16 CTAs per SM in all (four waves of four 8-warp CTAs), so the hardware's
// CTA scheduling evens out the last wave, and at least one 32-token group per warp in every
// CTA.
int nf4_splits(int bh, int n_groups) {
  const int want = (16 * sm_count() + bh - 1) / bh;
  return std::max(1, std::min(std::min(want, n_groups / kNf4DecWarps), kNf4MaxSplits));
}

// Block-GTQ decode: splits of whole 128-token chunks, at most one CTA per SM in total (a
// second partial wave would double the time of the CTAs in it). A CTA's four warpgroups take
// its chunks in turn, so its time is set by ceil(chunks / 4); the fewest splits that keep that
// number are used, which leaves the time as it is and makes the split merge smaller.
constexpr int kMaxGtqSplits = kMergeMax * kMergeMax;
// Upper bound of the split count for any length up to n_tiles tiles (it grows with n_tiles):
// the decode workspace is sized with it, so one workspace serves every length of a cache.
int gtq_splits_max(int bh, int n_tiles) {
  const int n_chunks = (n_tiles + kChunkTiles - 1) / kChunkTiles;
  return std::max(1, std::min(std::min(sm_count() / bh, n_chunks), kMaxGtqSplits));
}
int gtq_splits(int bh, int n_tiles) {
  const int n_chunks = (n_tiles + kChunkTiles - 1) / kChunkTiles;
  if (n_chunks == 0) return 1;                              // recent tokens only
  const int most = gtq_splits_max(bh, n_tiles);
  const int per_wg = (n_chunks + kDecWG * most - 1) / (kDecWG * most);
  return std::max(1, (n_chunks + kDecWG * per_wg - 1) / (kDecWG * per_wg));
}

struct DecodeWs {
  size_t tickets, part_m, part_l, part_o, total;
};

// Workspace of the decode kernels: tickets (`ticket_stride` counters per row: one final
// counter, then one per merge group), then (m, l, O) partials for `entries` entries per row,
// starting no earlier than `part_base`. The ticket region of a workspace must not move between
// calls: the last CTA returns every counter it used to zero, and a counter that once held a
// partial would start a later call at a wrong count.
DecodeWs decode_ws_layout(int bh, int entries, int rows, int ticket_stride, size_t part_base = 0) {
  DecodeWs w;
  w.tickets = sizeof(WsHeader);
  w.part_m = std::max<size_t>(align_up(w.tickets + 4ull * bh * ticket_stride, 128), part_base);
  w.part_l = align_up(w.part_m + 4ull * bh * entries * rows, 128);
  w.part_o = align_up(w.part_l + 4ull * bh * entries * rows, 128);
  w.total = align_up(w.part_o + 4ull * bh * entries * rows * kD, 128);
  return w;
}

// Merge of `splits` partials: groups of group_size splits, n_groups of them (1: one level).
struct MergePlan {
  int group_size, n_groups;
};
// Split merge plan: one level (the last CTA merges every split) while that takes at most two
// batched round trips to L2; above that, groups of about sqrt(splits), so each level is one.
MergePlan merge_plan(int splits) {
  if (splits <= 2 * kMergeBatch) return MergePlan{splits, 1};
  int gs = 1;
  while (gs * gs < splits) ++gs;
  return MergePlan{gs, (splits + gs - 1) / gs};
}

// Tickets per row for a cache: one final counter plus the merge groups of the largest split
// count any of its lengths uses, so the ticket region stays put for every call on the cache.
int gtq_ticket_stride(int bh, int capacity_tiles) {
  return 1 + merge_plan(gtq_splits_max(bh, capacity_tiles)).n_groups;
}
DecodeWs gtq_ws_layout(int bh, int splits, int ticket_stride, size_t part_base = 0) {
  const MergePlan mp = merge_plan(splits);
  return decode_ws_layout(bh, splits + mp.n_groups, 8, ticket_stride, part_base);
}

// Per-device attribute memos: atomics, so host threads calling in at once read either 0 (and
// query the attribute themselves) or the stored value.
int sm_count() {
  static std::atomic<int> cached[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Launches `kern` with programmatic stream serialization: it may begin (barrier setup, its
// own tables) while the previous kernel in the stream finishes; the kernels wait for that
// grid before they touch the caller's memory.
template <typename... P, typename... A>
cudaError_t launch_pdl(void (*kern)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}

kvq_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? KVQ_OK : cuda_fail(e);
}

Nf4Layout nf4_layout(int batch, int n_heads, int capacity) {
  Nf4Layout L;
  L.nblk = n_heads * kD / KVQ_NF4_BLOCK;
  L.t_pad = (capacity + KVQ_NF4_PAD - 1) / KVQ_NF4_PAD * KVQ_NF4_PAD;
  L.codes_bytes = static_cast<size_t>(batch) * L.nblk * L.t_pad * 128;
  return L;
}

// Opt-in shared memory per block of the current device (227 KB on a B200).
size_t max_smem() {
  static std::atomic<int> cached[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 227 * 1024;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (n <= 0) n = 227 * 1024;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return static_cast<size_t>(n);
}

// Chunk stages per warpgroup (1..4) that fit in shared memory; cbytes = bytes of one chunk stage.
int decode_stages(int cbytes) {
  const size_t per = static_cast<size_t>(kDecWG) * cbytes;
  const size_t room = max_smem() - decode_stage_off();
  return static_cast<int>(std::max<size_t>(1, std::min<size_t>(kStagesMax, room / per)));
}

size_t decode_smem_bytes(int cbytes) {
  const size_t stage = static_cast<size_t>(kDecWG) * cbytes * decode_stages(cbytes);
  // the stage area also holds the warpgroups' results at the end (kDecWG x 8 x 128 floats)
  return decode_stage_off() + std::max<size_t>(stage, static_cast<size_t>(kDecWG) * 8 * kD * sizeof(float));
}

// Test hooks (kvq_debug_decode): bounded-wait limit and the no-copy switch of the next decodes.
std::atomic<uint32_t> g_wait_limit{2000};   // test hook settings (kvq_debug_decode)
std::atomic<int> g_debug_no_loads{0};

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
    case KVQ_ERR_MISMATCH: return "packed cache does not match the descriptor or allocation";
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

size_t kvq_packed_header_bytes(int n_kv_heads) { return n_kv_heads >= 1 ? header_bytes(n_kv_heads) : 0; }

size_t kvq_packed_bytes(const kvq_cache_desc* c) {
  if (!cache_ok(c)) return 0;
  return header_bytes(c->n_kv_heads) +
         static_cast<size_t>(c->batch) * c->n_kv_heads * n_tiles_of(c->capacity) * tile_record_bytes(c->bits_k, c->bits_v);
}

size_t kvq_decode_workspace_bytes(const kvq_cache_desc* c, int n_q_heads) {
  if (!cache_ok(c) || n_q_heads < 1) return 0;
  const int bh = c->batch * c->n_kv_heads;
  const int cap_tiles = n_tiles_of(c->capacity);
  return gtq_ws_layout(bh, gtq_splits_max(bh, cap_tiles), gtq_ticket_stride(bh, cap_tiles)).total;
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
  { const cudaError_t e_ = cudaMemcpyAsync(&code, ws, sizeof(code), cudaMemcpyDeviceToHost, s); if (e_ != cudaSuccess) return cuda_fail(e_); }
  { const cudaError_t e_ = cudaStreamSynchronize(s); if (e_ != cudaSuccess) return cuda_fail(e_); }
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
  cudaError_t le;
  switch (kd->dtype) {
    case KVQ_F32:
      le = launch_pdl(kvq_calib_reduce<KVQ_F32>, grid, dim3(threads), 0, s, static_cast<const float*>(K), n_calib,
                      kd->stride_b, kd->stride_h, kd->stride_t, static_cast<int>(N), n_chunks, cws);
      break;
    case KVQ_F16:
      le = launch_pdl(kvq_calib_reduce<KVQ_F16>, grid, dim3(threads), 0, s, static_cast<const __half*>(K), n_calib,
                      kd->stride_b, kd->stride_h, kd->stride_t, static_cast<int>(N), n_chunks, cws);
      break;
    default:
      le = launch_pdl(kvq_calib_reduce<KVQ_BF16>, grid, dim3(threads), 0, s, static_cast<const __nv_bfloat16*>(K),
                      n_calib, kd->stride_b, kd->stride_h, kd->stride_t, static_cast<int>(N), n_chunks, cws);
  }
  if (le != cudaSuccess) return cuda_fail(le);
  le = launch_pdl(kvq_greedy_alloc, dim3(kd->n_heads), dim3(512), 0, s, static_cast<const double*>(cws.energy),
                  p->bits_k, p->w_max, p->mode, static_cast<kvq_head_alloc*>(alloc_out));
  if (le != cudaSuccess) return cuda_fail(le);
  return launch_status();
}

namespace {

// Quantizes tokens t_begin .. t_begin + kd->seq_len - 1 (input row i = token t_begin + i) into
// their tiles of `packed`; the rest of a partly covered first tile keeps its stored codes.
kvq_status launch_quant(const void* K, const kvq_tensor4* kd, const void* V, const kvq_tensor4* vd, const void* alloc,
                        const kvq_cache_desc* c, int t_begin, void* packed, void* stream) {
  kvq_status st;
  if ((st = check_tensor(K, kd)) != KVQ_OK) return st;
  if (!alloc || !packed || !aligned16(packed)) return KVQ_ERR_ARG;
  if (!cache_ok(c)) return KVQ_ERR_ARG;
  const bool keys_only = c->bits_v == 0;
  if (!keys_only) {
    if ((st = check_tensor(V, vd)) != KVQ_OK) return st;
    if (vd->dtype != kd->dtype || vd->batch != kd->batch || vd->n_heads != kd->n_heads || vd->seq_len != kd->seq_len)
      return KVQ_ERR_SHAPE;
  }
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
  QHeader qh;
  qh.mode = t_begin == 0 ? 1 : 2;
  qh.batch = c->batch;
  qh.capacity = c->capacity;
  qh.hdr_bytes = static_cast<int>(header_bytes(c->n_kv_heads));
  const int64_t vsb = keys_only ? 0 : vd->stride_b, vsh = keys_only ? 0 : vd->stride_h, vst = keys_only ? 0 : vd->stride_t;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Persistent grid: exactly the CTAs that are resident at once (registers and shared memory
  // both limit it), so every warp starts at launch and the tiles are spread evenly.
  // The shared-memory opt-in and the occupancy query are made once per device, dtype and value
  // width (they cost host time comparable to a small launch, e.g. a one-token append).
  static std::mutex occ_mu;
  static int occ[kMaxDevices][27] = {};
  static uint64_t occ_ctx[kMaxDevices][27] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
  const uint64_t ctx = context_id();
#define KVQ_LAUNCH_QUANT(DT, TY, BV)                                                                              \
  do {                                                                                                            \
    auto kern = kvq_quant_pack<DT, BV>;                                                                           \
    int per_sm = 0;                                                                                               \
    {                                                                                                             \
      std::lock_guard<std::mutex> lock(occ_mu);                                                                   \
      if (occ_ctx[dev][DT * 9 + BV] != ctx) {                                                                     \
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=    \
            cudaSuccess)                                                                                          \
          return KVQ_ERR_CUDA;                                                                                    \
        int n = 0;                                                                                                \
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, qw * 32, smem) != cudaSuccess)                \
          return KVQ_ERR_CUDA;                                                                                    \
        occ[dev][DT * 9 + BV] = std::max(1, n);                                                                   \
        occ_ctx[dev][DT * 9 + BV] = ctx;                                                                          \
      }                                                                                                           \
      per_sm = occ[dev][DT * 9 + BV];                                                                             \
    }                                                                                                             \
    const long long want = (n_tasks + qw - 1) / qw;                                                             \
    const unsigned grid =                                                                                         \
        static_cast<unsigned>(std::min<long long>(want, static_cast<long long>(sm_count()) * std::max(1, per_sm))); \
    const cudaError_t le = launch_pdl(kern, dim3(grid), dim3(qw * 32), smem, s, static_cast<const TY*>(K),         \
                                      kd->stride_b, kd->stride_h, kd->stride_t, static_cast<const TY*>(V), vsb,  \
                                      vsh, vst, t_begin, t_end, tile_lo, n_tiles, c->n_kv_heads, tiles_cap,      \
                                      static_cast<const kvq_head_alloc*>(alloc), c->bits_k, c->bits_v,           \
                                      static_cast<uint8_t*>(packed), rec, static_cast<int>(n_tasks), qh);        \
    if (le != cudaSuccess) return cuda_fail(le);                                                                  \
  } while (0)
#define KVQ_QUANT_BV(DT, TY)                                                                                      \
  switch (c->bits_v) {                                                                                            \
    case 0: KVQ_LAUNCH_QUANT(DT, TY, 0); break;                                                                   \
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

}  // extern "C"
namespace {

// Checks a [batch][n_kv_heads][>= n][128] view against a cache descriptor.
kvq_status check_kv_view(const void* p, const kvq_tensor4* t, const kvq_cache_desc* c, int n) {
  kvq_status st = check_tensor(p, t);
  if (st != KVQ_OK) return st;
  if (t->batch != c->batch || t->n_heads != c->n_kv_heads || t->seq_len < n) return KVQ_ERR_SHAPE;
  return KVQ_OK;
}

kvq_status launch_decode(const void* q, const kvq_tensor4* qd, const void* packed, const void* alloc,
                         const kvq_cache_desc* c, int seq_len, const kvq_decode_extra* ex, float* out, void* ws,
                         size_t ws_bytes, void* stream, size_t part_base = 0) {
  kvq_status st;
  if ((st = check_tensor(q, qd)) != KVQ_OK) return st;
  if (!packed || !alloc || !out || !aligned16(packed) || !aligned16(alloc)) return KVQ_ERR_ARG;
  if (!cache_ok(c)) return KVQ_ERR_ARG;
  if (qd->seq_len != 1 || qd->batch != c->batch) return KVQ_ERR_SHAPE;
  if (qd->n_heads % c->n_kv_heads != 0 || qd->n_heads / c->n_kv_heads > 8) return KVQ_ERR_UNSUPPORTED;
  const bool keys_only = c->bits_v == 0;
  const bool dense_v = ex && ex->V;
  const int n_recent = (ex && ex->K_recent) ? ex->krd.seq_len : 0;
  if (keys_only != dense_v) return keys_only ? KVQ_ERR_UNSUPPORTED : KVQ_ERR_ARG;
  if (ex && (ex->K_recent != nullptr) != (ex->V_recent != nullptr)) return KVQ_ERR_ARG;
  if (seq_len < (n_recent > 0 ? 0 : 1) || seq_len > c->capacity) return KVQ_ERR_RANGE;
  if (dense_v) {
    if ((st = check_kv_view(ex->V, &ex->vd, c, seq_len)) != KVQ_OK) return st;
    if (ex->vd.dtype != KVQ_BF16 && ex->vd.dtype != KVQ_F16) return KVQ_ERR_DTYPE;
  }
  if (n_recent > 0) {
    if ((st = check_kv_view(ex->K_recent, &ex->krd, c, n_recent)) != KVQ_OK) return st;
    if ((st = check_kv_view(ex->V_recent, &ex->vrd, c, n_recent)) != KVQ_OK) return st;
  }
  const int bh = c->batch * c->n_kv_heads;
  const int n_tiles = n_tiles_of(seq_len);
  const int splits = gtq_splits(bh, n_tiles);
  const MergePlan mp = merge_plan(splits);
  const int ticket_stride = gtq_ticket_stride(bh, n_tiles_of(c->capacity));
  const DecodeWs L = gtq_ws_layout(bh, splits, ticket_stride, part_base);
  if (!ws || ws_bytes < L.total || !aligned16(ws) || ws_bytes < kvq_decode_workspace_bytes(c, qd->n_heads))
    return KVQ_ERR_WORKSPACE;
  if ((st = ensure_tables()) != KVQ_OK) return st;
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  const int rec = static_cast<int>(tile_record_bytes(c->bits_k, c->bits_v));
  const int cb = chunk_bytes(rec) + (dense_v ? kChunkTokens * 2 * kD : 0);
  const size_t smem = decode_smem_bytes(cb);
  // one chunk stage per warpgroup must fit (keys-only caches above 4 bits per dim do not)
  if (smem > max_smem()) return KVQ_ERR_UNSUPPORTED;
  DecArgs a{};
  a.q = q;
  a.qsb = qd->stride_b;
  a.qsh = qd->stride_h;
  a.q_dtype = qd->dtype;
  a.n_q_heads = qd->n_heads;
  a.n_kv_heads = c->n_kv_heads;
  a.batch = c->batch;
  if (dense_v) {
    a.v_dense = ex->V;
    a.vsb = ex->vd.stride_b;
    a.vsh = ex->vd.stride_h;
    a.vst = ex->vd.stride_t;
  }
  a.cbytes = cb;
  if (n_recent > 0) {
    a.k_rec = ex->K_recent;
    a.v_rec = ex->V_recent;
    a.krsb = ex->krd.stride_b;
    a.krsh = ex->krd.stride_h;
    a.krst = ex->krd.stride_t;
    a.vrsb = ex->vrd.stride_b;
    a.vrsh = ex->vrd.stride_h;
    a.vrst = ex->vrd.stride_t;
    a.kr_dtype = ex->krd.dtype;
    a.vr_dtype = ex->vrd.dtype;
    a.n_recent = n_recent;
  }
  a.packed = static_cast<const uint8_t*>(packed);
  a.alloc = static_cast<const kvq_head_alloc*>(alloc);
  a.hdr_bytes = static_cast<int>(header_bytes(c->n_kv_heads));
  a.tiles_cap = n_tiles_of(c->capacity);
  a.rec_bytes = rec;
  a.bits_k = c->bits_k;
  a.bits_v = c->bits_v;
  a.capacity = c->capacity;
  a.seq_len = seq_len;
  a.splits = splits;
  a.n_groups = splits > 1 ? mp.n_groups : 0;
  a.group_size = mp.group_size;
  a.n_stages = decode_stages(cb);
  a.out = out;
  a.part_m = reinterpret_cast<float*>(w8 + L.part_m);
  a.part_l = reinterpret_cast<float*>(w8 + L.part_l);
  a.part_o = reinterpret_cast<float*>(w8 + L.part_o);
  a.tickets = reinterpret_cast<unsigned*>(w8 + L.tickets);
  a.ticket_stride = ticket_stride;
  a.status = reinterpret_cast<unsigned*>(w8);
  a.wait_limit = g_wait_limit.load(std::memory_order_relaxed);
  a.debug_no_loads = g_debug_no_loads.load(std::memory_order_relaxed);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  dim3 grid(splits, bh);
  const int vm = dense_v ? (ex->vd.dtype == KVQ_BF16 ? kDenseBf16 : kDenseF16) : c->bits_v;
  // The shared-memory opt-in is raised once per device and value mode to the largest size
  // launched so far (the call costs host time comparable to the launch itself).
  static std::mutex smem_mu;
  static int smem_set[kMaxDevices][kDenseF16 + 1] = {};
  static uint64_t smem_ctx[kMaxDevices][kDenseF16 + 1] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
  const uint64_t ctx = context_id();
#define KVQ_LAUNCH_DEC(VM)                                                                                            \
  do {                                                                                                                \
    auto kern = kvq_decode_gtq<VM>;                                                                                   \
    {                                                                                                                 \
      std::lock_guard<std::mutex> lock(smem_mu);                                                                      \
      if (smem_ctx[dev][VM] != ctx || smem_set[dev][VM] < static_cast<int>(smem)) {                                  \
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,                 \
                                                   static_cast<int>(smem));                                           \
        if (e != cudaSuccess) return cuda_fail(e);                                                                    \
        smem_set[dev][VM] = static_cast<int>(smem);                                                                   \
        smem_ctx[dev][VM] = ctx;                                                                                      \
      }                                                                                                               \
    }                                                                                                                 \
    const cudaError_t le = launch_pdl(kern, grid, dim3(kDecThreads), smem, s, a);                                     \
    if (le != cudaSuccess) return cuda_fail(le);                                                                      \
  } while (0)
  switch (vm) {
    case 1: KVQ_LAUNCH_DEC(1); break;
    case 2: KVQ_LAUNCH_DEC(2); break;
    case 3: KVQ_LAUNCH_DEC(3); break;
    case 4: KVQ_LAUNCH_DEC(4); break;
    case 5: KVQ_LAUNCH_DEC(5); break;
    case 6: KVQ_LAUNCH_DEC(6); break;
    case 7: KVQ_LAUNCH_DEC(7); break;
    case 8: KVQ_LAUNCH_DEC(8); break;
    case kDenseBf16: KVQ_LAUNCH_DEC(kDenseBf16); break;
    default: KVQ_LAUNCH_DEC(kDenseF16); break;
  }
#undef KVQ_LAUNCH_DEC
  return launch_status();
}

}  // namespace
extern "C" {

kvq_status kvq_decode_attn(const void* q, const kvq_tensor4* qd, const void* packed, const void* alloc,
                           const kvq_cache_desc* c, int seq_len, float* out, void* ws, size_t ws_bytes,
                           void* stream) {
  return launch_decode(q, qd, packed, alloc, c, seq_len, nullptr, out, ws, ws_bytes, stream);
}

kvq_status kvq_decode_attn_ex(const void* q, const kvq_tensor4* qd, const void* packed, const void* alloc,
                              const kvq_cache_desc* c, int seq_len, const kvq_decode_extra* extra, float* out,
                              void* ws, size_t ws_bytes, void* stream) {
  return launch_decode(q, qd, packed, alloc, c, seq_len, extra, out, ws, ws_bytes, stream);
}

kvq_status kvq_packed_status(const void* packed, void* stream, int* device_code) {
  if (!packed) return KVQ_ERR_ARG;
  unsigned int code = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint8_t* p = static_cast<const uint8_t*>(packed) + offsetof(kvq_packed_header, status);
  { const cudaError_t e_ = cudaMemcpyAsync(&code, p, sizeof(code), cudaMemcpyDeviceToHost, s); if (e_ != cudaSuccess) return cuda_fail(e_); }
  { const cudaError_t e_ = cudaStreamSynchronize(s); if (e_ != cudaSuccess) return cuda_fail(e_); }
  if (device_code) *device_code = static_cast<int>(code);
  return code == 0 ? KVQ_OK : static_cast<kvq_status>(code);
}

const char* kvq_last_cuda_error(void) {
  return cudaGetErrorString(static_cast<cudaError_t>(g_last_cuda_error.load()));
}

kvq_status kvq_debug_decode(int wait_limit, int no_loads) {
  if (wait_limit < 1) return KVQ_ERR_ARG;
  g_wait_limit.store(static_cast<uint32_t>(wait_limit), std::memory_order_relaxed);
  g_debug_no_loads.store(no_loads ? 1 : 0, std::memory_order_relaxed);
  return KVQ_OK;
}

size_t kvq_nf4_packed_bytes(int batch, int n_heads, int capacity, int head_dim) {
  if (batch < 1 || n_heads < 2 || (n_heads & 1) || capacity < 1 || head_dim != kD) return 0;
  const Nf4Layout L = nf4_layout(batch, n_heads, capacity);
  return 2 * L.codes_bytes + 2 * (L.codes_bytes / 128) * sizeof(__half);
}

size_t kvq_nf4_decode_workspace_bytes(int batch, int n_heads, int capacity, int head_dim) {
  if (batch < 1 || n_heads < 1 || capacity < 1 || head_dim != kD) return 0;
  const int bh = batch * n_heads;
  return decode_ws_layout(bh, nf4_splits(bh, (capacity + 31) / 32), 1, 1).total;
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
  const DecodeWs Lw = decode_ws_layout(bh, splits, 1, 1);
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
// holds until the process exits. Its device address is looked up on every call (with the
// caller's device current) and handed to the ordinary Block-GTQ decode kernel as its
// workspace.
namespace {

constexpr size_t kNoAllocScratchBytes = 2u << 20;   // 2 MiB per device
constexpr size_t kNoAllocTicketBytes = 64 * 1024;   // status word and split tickets of every call
__device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device. When the address is new for
// this device (its first call, or a context created again after a reset), the array is zeroed
// by an asynchronous memset on the caller's stream, so the decode launched next on that
// stream sees zero split tickets and a clear status word; the kernel returns the tickets to
// zero after every call.
kvq_status decode_scratch(cudaStream_t s, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return KVQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] != p) {
    { const cudaError_t e_ = cudaMemsetAsync(p, 0, kNoAllocScratchBytes, s); if (e_ != cudaSuccess) return cuda_fail(e_); }
    g_scratch_ptr[dev] = p;
  }
  *out = p;
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
  // Split tickets live in a fixed area at the start of the array, so calls on caches of any
  // shape use counters that the previous calls returned to zero; the partials follow it.
  const int bh = cache->batch * cache->n_kv_heads;
  const int cap_tiles = n_tiles_of(cache->capacity);
  const int stride = gtq_ticket_stride(bh, cap_tiles);
  if (sizeof(WsHeader) + 4ull * bh * stride > kNoAllocTicketBytes) return KVQ_ERR_WORKSPACE;
  if (gtq_ws_layout(bh, gtq_splits_max(bh, cap_tiles), stride, kNoAllocTicketBytes).total > kNoAllocScratchBytes)
    return KVQ_ERR_WORKSPACE;
  kvq_status st = ensure_tables();
  if (st != KVQ_OK) return st;
  void* scratch = nullptr;
  if ((st = decode_scratch(static_cast<cudaStream_t>(stream), &scratch)) != KVQ_OK) return st;
  return launch_decode(q, qd, packed, alloc, cache, seq_len, nullptr, out, scratch, kNoAllocScratchBytes, stream,
                       kNoAllocTicketBytes);
}

kvq_status kvq_decode_noalloc_status(void* stream, int* device_code) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  kvq_status st = decode_scratch(s, &scratch);
  if (st != KVQ_OK) return st;
  unsigned int code = 0;
  { const cudaError_t e_ = cudaMemcpyAsync(&code, scratch, sizeof(code), cudaMemcpyDeviceToHost, s); if (e_ != cudaSuccess) return cuda_fail(e_); }
  { const cudaError_t e_ = cudaStreamSynchronize(s); if (e_ != cudaSuccess) return cuda_fail(e_); }
  if (code != 0) {
    { const cudaError_t e_ = cudaMemsetAsync(scratch, 0, sizeof(code), s); if (e_ != cudaSuccess) return cuda_fail(e_); }
    { const cudaError_t e_ = cudaStreamSynchronize(s); if (e_ != cudaSuccess) return cuda_fail(e_); }
  }
  if (device_code) *device_code = static_cast<int>(code);
  return code == 0 ? KVQ_OK : static_cast<kvq_status>(code);
}

}  // extern "C"
