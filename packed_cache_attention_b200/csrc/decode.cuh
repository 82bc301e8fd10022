// Fused decode attention read straight from the packed Block-GTQ cache (page "RoPE-aware bit
// allocation for KV cache quantization", abstract: attention served from the packed cache;
// the NQKV review's editorial extensions propose folding the table lookup into attention).
//
// Grid: (splits, batch * n_kv_heads). Each CTA owns a contiguous range of 128-token chunks
// (4 tile records) of one (sequence, KV head) and runs a pipeline over them:
//   load warp     bulk-copies each chunk's tile records into a shared-memory stage;
//   16 warps      dequantize codes through shared-memory lookup tables straight into tensor
//                 memory: K-hat rows (lane = token, one fp16 pair per column) and V-hat^T
//                 rows (lane = dim, columns = token pairs); then run the softmax;
//   MMA warp      one thread issues tcgen05.mma (M = 128, N = 16, fp16 -> fp32):
//                   S^T[128 tokens][16]  = Khat[128][K cols]  x  Q'^T  (Q' hi rows 0-7, lo 8-15)
//                   O^T[128 dims][16]   = Vhat^T[128][128]   x  P'^T  (P' hi rows 0-7, lo 8-15)
// with K-hat and V-hat^T as the A operand in tensor memory and Q', P' as the small B operand
// in shared memory. K columns follow the stream order of the tile layout (width classes,
// each padded to whole groups of 4 block pairs); Q' carries f_b, log2(e)/sqrt(d) and a per
// query power of two that keeps its fp16 split in range, and the key norm scales S after
// the MMA. Softmax runs online in the log2 domain with P' = p * vnorm / sqrt(d) split into
// fp16 hi + lo. Warp group g handles query rows 2g, 2g+1 of the softmax and of O.
// Tensor memory and shared buffers are double-buffered by chunk parity; every hand-off is
// an mbarrier with a bounded wait.
// Splits write (m, l, O) partials to the workspace; the last CTA of each group of 8 splits
// merges its group, and the last group merges the groups (atomic tickets), writing
// out = O / l.
#pragma once

#include "common.cuh"
#include "tcgen05.cuh"

namespace kvq {

constexpr int kDecComputeWarps = 16;
constexpr int kDecMmaWarp = 16;
constexpr int kDecLoadWarp = 17;
constexpr int kDecThreads = 18 * 32;
constexpr int kChunkTiles = 4;
constexpr int kChunkTokens = kChunkTiles * kTile;   // = MMA M = tensor-memory lanes
constexpr int kDecStagesMax = 4;
constexpr int kMaxMergeSplits = 160;
constexpr int kMergeGroup = 8;       // splits merged by the last CTA of each group (first level)
constexpr int kTargetCtas = 148;     // one CTA per SM on a 148-SM B200
constexpr int kGroupPairs = 4;       // block pairs (tensor-memory columns) per K decode group
constexpr int kMaxKGroups = 32;      // at most 64 / 4 + 8 groups per head
constexpr uint32_t kWaitLimit = 1u << 20;

// Tensor-memory columns (512 allocated): A_K[2] (128 each), A_V[2] (64 each), S[2], O[2] (16 each).
constexpr uint32_t kTmemCols = 512;
__device__ __forceinline__ uint32_t col_ak(int b) { return 128u * b; }
__device__ __forceinline__ uint32_t col_av(int b) { return 256u + 64u * b; }
__device__ __forceinline__ uint32_t col_s(int b) { return 384u + 16u * b; }
__device__ __forceinline__ uint32_t col_o(int b) { return 416u + 16u * b; }

// Shared-memory map (byte offsets from the start of dynamic shared memory).
// Pair tables give the fp16 pair {c[i & m], c[i >> w]} for the 2w-bit index i of two
// consecutive codes. Widths 1..3 keep one copy per lane (entry e of lane l at word 32 e + l)
// so that 32 lanes never conflict; widths 4..6 keep one copy; widths 7, 8 use single-code
// fp16 tables.
__host__ __device__ constexpr int lut_off(int w) {
  return w == 1 ? 0 : w == 2 ? 512 : w == 3 ? 2560 : w == 4 ? 10752 : w == 5 ? 11776 : w == 6 ? 15872 : w == 7 ? 32256
                                                                                                             : 32512;
}
constexpr int kCentOff = 33024;                 // 510 fp16 centroids
constexpr int kBQOff = 34048;                   // Q' (B operand of S), K-major, up to 256 K elements
constexpr int kBQBytes = 32 * 256;
constexpr int kBPOff = kBQOff + kBQBytes;       // P' (B operand of O), 2 buffers, N-major
constexpr int kBPBytes = 4096;
constexpr int kHdrOff = kBPOff + 2 * kBPBytes;

struct DecHeader {
  uint64_t full[kDecStagesMax];
  uint64_t empty[kDecStagesMax];
  uint64_t kready[2], vready[2], pready[2], sfull[2], ofull[2];
  uint32_t tmem_base;
  int k_cols;                        // K columns used by the S MMA (multiple of 8)
  int n_kgroups[4];
  uint32_t kgroup[4][kMaxKGroups];   // width | bit offset << 4 | column << 16
  int8_t col_block[128];             // block of K column c (-1 = padding)
  float qscale[8];                   // 2^e that undoes the range scaling of Q' row h
  float xmax[2][4][4][2];            // chunk max: [parity][warp group][quarter][query]
  float lpart[4][4][2];              // row sums: [warp group][quarter][query]
  int last;
  float mw[8][kMaxMergeSplits];      // cross-split merge: weight 2^(m_s - M) per head and member
  float Lsum[8];
  float Mmax[8];
};

__host__ __device__ constexpr int decode_stage_off() { return kHdrOff + ((static_cast<int>(sizeof(DecHeader)) + 127) / 128) * 128; }

// ---------------------------------------------------------------- code extraction + lookup

// Bits [p, p + n) of the 64-bit value hi:lo (p, n constant after unrolling, n <= 16).
__device__ __forceinline__ uint32_t field(uint32_t lo, uint32_t hi, int p, int n) {
  uint32_t v;
  if (p >= 32) v = hi >> (p - 32);
  else if (p + n <= 32) v = lo >> p;
  else v = __funnelshift_r(lo, hi, p);
  return v & ((1u << n) - 1u);
}

// fp16 pair for the pair index idx = code_a | code_b << W (code_a in the low half).
template <int W>
__device__ __forceinline__ uint32_t pair_value(uint32_t idx, const uint8_t* sm, uint32_t lane4) {
  if constexpr (W <= 3) {
    return *reinterpret_cast<const uint32_t*>(sm + lut_off(W) + ((idx << 7) | lane4));
  } else if constexpr (W <= 6) {
    return *reinterpret_cast<const uint32_t*>(sm + lut_off(W) + (idx << 2));
  } else {
    const uint16_t* t = reinterpret_cast<const uint16_t*>(sm + lut_off(W));
    return static_cast<uint32_t>(t[idx & ((1u << W) - 1u)]) | (static_cast<uint32_t>(t[idx >> W]) << 16);
  }
}

// One K decode group: 4 consecutive block pairs of width W whose first code starts at bit
// `off` of this lane's token stream; kw points at word 0 of the token (word i at kw[32 i]).
template <int W>
__device__ __forceinline__ void k_group(const uint32_t* kw, uint32_t off, uint32_t taddr, const uint8_t* sm,
                                        uint32_t lane4) {
  const uint32_t j0 = off >> 5, s = off & 31u;
  const uint32_t x0 = kw[j0 * 32], x1 = kw[(j0 + 1) * 32];
  const uint32_t x2 = (W >= 5) ? kw[(j0 + 2) * 32] : 0u;
  const uint32_t r0 = __funnelshift_r(x0, x1, s);
  const uint32_t r1 = __funnelshift_r(x1, x2, s);
  uint32_t v[kGroupPairs];
#pragma unroll
  for (int k = 0; k < kGroupPairs; ++k) v[k] = pair_value<W>(field(r0, r1, 2 * W * k, 2 * W), sm, lane4);
  tc::tmem_st<kGroupPairs>(taddr, v);
}

// V-hat^T row of one dim for one tile: 16 token pairs (2u, 2u+1) -> 16 columns.
template <int BV>
__device__ __forceinline__ void v_tile(const uint32_t* vw, uint32_t taddr, const uint8_t* sm, uint32_t lane4) {
  uint32_t x[BV + 1];
#pragma unroll
  for (int i = 0; i < BV; ++i) x[i] = vw[i * kD];
  x[BV] = 0u;
  uint32_t v[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int p = 2 * BV * u;
    v[u] = pair_value<BV>(field(x[p >> 5], x[(p >> 5) + 1], p & 31, 2 * BV), sm, lane4);
  }
  tc::tmem_st<16>(taddr, v);
}

__device__ __forceinline__ void k_group_any(int w, const uint32_t* kw, uint32_t off, uint32_t taddr,
                                            const uint8_t* sm, uint32_t lane4) {
  switch (w) {
    case 1: k_group<1>(kw, off, taddr, sm, lane4); break;
    case 2: k_group<2>(kw, off, taddr, sm, lane4); break;
    case 3: k_group<3>(kw, off, taddr, sm, lane4); break;
    case 4: k_group<4>(kw, off, taddr, sm, lane4); break;
    case 5: k_group<5>(kw, off, taddr, sm, lane4); break;
    case 6: k_group<6>(kw, off, taddr, sm, lane4); break;
    case 7: k_group<7>(kw, off, taddr, sm, lane4); break;
    default: k_group<8>(kw, off, taddr, sm, lane4); break;
  }
}

__device__ __forceinline__ void v_tile_any(int bv, const uint32_t* vw, uint32_t taddr, const uint8_t* sm,
                                           uint32_t lane4) {
  switch (bv) {
    case 1: v_tile<1>(vw, taddr, sm, lane4); break;
    case 2: v_tile<2>(vw, taddr, sm, lane4); break;
    case 3: v_tile<3>(vw, taddr, sm, lane4); break;
    case 4: v_tile<4>(vw, taddr, sm, lane4); break;
    case 5: v_tile<5>(vw, taddr, sm, lane4); break;
    case 6: v_tile<6>(vw, taddr, sm, lane4); break;
    case 7: v_tile<7>(vw, taddr, sm, lane4); break;
    default: v_tile<8>(vw, taddr, sm, lane4); break;
  }
}

// Order-preserving map of fp32 to int32 (and back: the map is its own inverse).
__device__ __forceinline__ int ordered(float x) {
  const int i = __float_as_int(x);
  return i ^ ((i >> 31) & 0x7fffffff);
}
__device__ __forceinline__ float from_ordered(int i) { return __int_as_float(i ^ ((i >> 31) & 0x7fffffff)); }

__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

__device__ __forceinline__ void record_timeout(unsigned* status) { atomicCAS(status, 0u, static_cast<unsigned>(KVQ_ERR_TIMEOUT)); }

// ---------------------------------------------------------------- cross-split merge

// Merge the (m, l, O) partials first .. first+n-1 of (sequence, KV head) bh: into entry dst
// of the workspace (out == nullptr) or into out = O / l for the G real query heads. Called
// by every thread of the CTA; the 16 compute warps do the work.
__device__ __forceinline__ void merge_partials(DecHeader& S, uint8_t* scratch, int bh, int pitch, int first, int n,
                                               float* part_m, float* part_l, float* part_o, int dst, float* out,
                                               int G) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (warp < 8) {
    const int hg = warp;
    const size_t p0 = (static_cast<size_t>(bh) * pitch + first) * 8 + hg;
    float M = -INFINITY;
    for (int s = lane; s < n; s += 32) M = fmaxf(M, __ldcg(part_m + p0 + static_cast<size_t>(s) * 8));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.0f;
    for (int s = lane; s < n; s += 32) {
      const size_t pi = p0 + static_cast<size_t>(s) * 8;
      const float ms = __ldcg(part_m + pi);
      const float wt = (ms == -INFINITY) ? 0.0f : fast_exp2(ms - M);
      S.mw[hg][s] = wt;
      L += __ldcg(part_l + pi) * wt;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (lane == 0) {
      S.Lsum[hg] = L;
      S.Mmax[hg] = M;
    }
  }
  __syncthreads();
  // O: 256 (head, 4-dim) quads; threads 0..255 and 256..511 take halves of the member list.
  const int quad = tid & 255, half = tid >> 8;
  const int hg = quad >> 5, j4 = quad & 31;
  const int s_mid = n / 2;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  if (half < 2) {
    const int s0 = half ? s_mid : 0, s1 = half ? n : s_mid;
    const float4* po = reinterpret_cast<const float4*>(part_o);
#pragma unroll 4
    for (int s = s0; s < s1; ++s) {
      const float wt = S.mw[hg][s];
      const float4 v = __ldcg(po + ((static_cast<size_t>(bh) * pitch + first + s) * 8 + hg) * (kD / 4) + j4);
      o.x += v.x * wt; o.y += v.y * wt; o.z += v.z * wt; o.w += v.w * wt;
    }
  }
  float4* red = reinterpret_cast<float4*>(scratch);
  if (half == 1) red[quad] = o;
  __syncthreads();
  if (half == 0) {
    const float4 v = red[quad];
    o.x += v.x; o.y += v.y; o.z += v.z; o.w += v.w;
    if (out != nullptr) {
      if (hg < G) {
        const float inv = 1.0f / S.Lsum[hg];
        reinterpret_cast<float4*>(out + static_cast<size_t>(hg) * kD)[j4] =
            make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
      }
    } else {
      const size_t pd = (static_cast<size_t>(bh) * pitch + dst) * 8 + hg;
      reinterpret_cast<float4*>(part_o + pd * kD)[j4] = o;
      if (j4 == 0) {
        part_m[pd] = S.Mmax[hg];
        part_l[pd] = S.Lsum[hg];
      }
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------- the kernel

template <int DT>
__global__ void __launch_bounds__(kDecThreads, 1) kvq_decode_gtq(
    const typename Elem<DT>::T* __restrict__ q, int64_t qsb, int64_t qsh, int n_q_heads, int n_kv_heads,
    const uint8_t* __restrict__ packed, const kvq_head_alloc* __restrict__ alloc, int tiles_cap, int rec_bytes,
    int bits_k, int bits_v, int seq_len, int splits, int n_groups, int n_stages, float* __restrict__ out,
    float* __restrict__ part_m, float* __restrict__ part_l, float* __restrict__ part_o,
    unsigned* __restrict__ tickets, unsigned* __restrict__ status) {
  extern __shared__ __align__(1024) uint8_t sm[];
  DecHeader& S = *reinterpret_cast<DecHeader*>(sm + kHdrOff);
  uint8_t* stages = sm + decode_stage_off();

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / n_kv_heads, hkv = bh % n_kv_heads;
  const int G = n_q_heads / n_kv_heads;
  const kvq_head_alloc* al = alloc + hkv;
  // An allocation made for another budget does not match the record size: write nothing.
  if (al->k_words != bits_k * kD || al->bits_k != bits_k) return;
  const int n_tiles = (seq_len + kTile - 1) / kTile;
  const int n_chunks_all = (n_tiles + kChunkTiles - 1) / kChunkTiles;
  const int c_begin = static_cast<int>((static_cast<long long>(split) * n_chunks_all) / splits);
  const int c_end = static_cast<int>((static_cast<long long>(split + 1) * n_chunks_all) / splits);
  const int n_chunks = c_end - c_begin;
  const int tile_end = min(n_tiles, c_end * kChunkTiles);
  const uint8_t* src = packed + static_cast<size_t>(bh) * tiles_cap * rec_bytes;
  const int stage_bytes = kChunkTiles * rec_bytes;
  const float inv_sqrt_d = 0.08838834764831845f;

  // ------------------------------------------------------------------ setup
  if (tid == 0) {
    for (int i = 0; i < kDecStagesMax; ++i) {
      tc::mbar_init(&S.full[i], 1);
      tc::mbar_init(&S.empty[i], kDecComputeWarps);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&S.kready[i], kDecComputeWarps);
      tc::mbar_init(&S.vready[i], kDecComputeWarps);
      tc::mbar_init(&S.pready[i], kDecComputeWarps);
      tc::mbar_init(&S.sfull[i], 1);
      tc::mbar_init(&S.ofull[i], 1);
    }
    tc::mbar_fence_init();
  }
  if (warp == kDecMmaWarp) tc::tmem_alloc(&S.tmem_base, kTmemCols);
  uint16_t* cent = reinterpret_cast<uint16_t*>(sm + kCentOff);
  for (int i = tid; i < kCentroidCount; i += blockDim.x) cent[i] = c_tab.centroid_f16[i];
  // K columns: classes in stream order, each padded to whole groups of 4 block pairs.
  if (tid == 0) {
    int col = 0, ng = 0;
    uint32_t groups[kMaxKGroups];
    for (int i = 0; i < 128; ++i) S.col_block[i] = -1;
    const int n_cls = min(max(al->n_classes, 0), 8);
    for (int c = 0; c < n_cls; ++c) {
      const int w = al->class_width[c], first = al->class_first[c], nb = al->class_blocks[c];
      const int bit = al->class_bit[c];
      for (int k0 = 0; k0 < nb && ng < kMaxKGroups; k0 += kGroupPairs) {
        groups[ng++] = static_cast<uint32_t>(w) | (static_cast<uint32_t>(bit + 2 * w * k0) << 4) |
                       (static_cast<uint32_t>(col) << 16);
        for (int k = 0; k < kGroupPairs && k0 + k < nb; ++k) S.col_block[col + k] = static_cast<int8_t>(al->stream_block[first + k0 + k]);
        col += kGroupPairs;
      }
    }
    S.k_cols = (col + 7) & ~7;
    // Balance the groups over the 4 warp groups (cost: 1 per pair lookup, 2 for the
    // single-code widths 7 and 8, plus the word loads).
    int load[4] = {0, 0, 0, 0};
    for (int g = 0; g < 4; ++g) S.n_kgroups[g] = 0;
    for (int i = 0; i < ng; ++i) {
      const int w = groups[i] & 15;
      const int cost = kGroupPairs * (w >= 7 ? 2 : 1) + 2 + (w >= 5 ? 1 : 0);
      int best = 0;
      for (int g = 1; g < 4; ++g)
        if (load[g] < load[best]) best = g;
      load[best] += cost;
      S.kgroup[best][S.n_kgroups[best]++] = groups[i];
    }
  }
  __syncthreads();
  // Lookup tables.
  for (int w = 1; w <= 3; ++w) {
    const int n = 1 << (2 * w);
    uint32_t* t = reinterpret_cast<uint32_t*>(sm + lut_off(w));
    for (int i = tid; i < n * 32; i += blockDim.x) {
      const int e = i >> 5;
      const uint16_t* c = cent + ((1 << w) - 2);
      t[i] = static_cast<uint32_t>(c[e & ((1 << w) - 1)]) | (static_cast<uint32_t>(c[e >> w]) << 16);
    }
  }
  for (int w = 4; w <= 6; ++w) {
    const int n = 1 << (2 * w);
    uint32_t* t = reinterpret_cast<uint32_t*>(sm + lut_off(w));
    const uint16_t* c = cent + ((1 << w) - 2);
    for (int e = tid; e < n; e += blockDim.x)
      t[e] = static_cast<uint32_t>(c[e & ((1 << w) - 1)]) | (static_cast<uint32_t>(c[e >> w]) << 16);
  }
  for (int w = 7; w <= 8; ++w) {
    uint16_t* t = reinterpret_cast<uint16_t*>(sm + lut_off(w));
    for (int e = tid; e < (1 << w); e += blockDim.x) t[e] = cent[(1 << w) - 2 + e];
  }
  // Q' rows: q_h * f_b * log2(e) / sqrt(d), scaled per row by 2^-e so the largest |Q'| is in
  // [0.5, 1); the MMA result is multiplied back by qscale[h] = 2^e.
  float* qtmp = reinterpret_cast<float*>(stages);   // [8][128] fp32, before the stages are used
  for (int i = tid; i < 8 * kD; i += blockDim.x) {
    const int hg = i / kD, j = i % kD;
    float v = 0.0f;
    if (hg < G) v = Elem<DT>::to_f32(q[b * qsb + (hkv * G + hg) * qsh + j]) * al->dequant[j % kH] * (inv_sqrt_d * kLog2e);
    qtmp[i] = v;
  }
  __syncthreads();
  if (warp < 8) {
    const int hg = warp;
    float mx = 0.0f;
    for (int j = lane; j < kD; j += 32) mx = fmaxf(mx, fabsf(qtmp[hg * kD + j]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    int e = 0;
    if (mx > 0.0f) frexpf(mx, &e);
    if (lane == 0) S.qscale[hg] = ldexpf(1.0f, e);
    const float sc = ldexpf(1.0f, -e);
    for (int j = lane; j < kD; j += 32) qtmp[hg * kD + j] *= sc;
  }
  __syncthreads();
  // B operand of S, K-major, no swizzle: element (n, k) at (k/8)*256 + (n/8)*128 + (n%8)*16 + (k%8)*2;
  // K element k = 2c + r is dim b + 64 r of the block in column c; n < 8: hi part of row n,
  // n >= 8: lo part of row n - 8.
  {
    const int k_elems = 2 * S.k_cols;
    for (int i = tid; i < 8 * k_elems; i += blockDim.x) {
      const int n = i / k_elems, k = i % k_elems;
      const int blk = S.col_block[k >> 1];
      __half hi = __float2half_rn(0.0f), lo = hi;
      if (blk >= 0) split_hilo(qtmp[n * kD + blk + kH * (k & 1)], hi, lo);
      const int base = (k >> 3) * 256 + (k & 7) * 2;
      *reinterpret_cast<__half*>(sm + kBQOff + base + n * 16) = hi;
      *reinterpret_cast<__half*>(sm + kBQOff + base + 128 + n * 16) = lo;
    }
  }
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = S.tmem_base;

  if (warp == kDecLoadWarp) {
    // ---------------------------------------------------------------- bulk loads
    if (lane == 0) {
      for (int i = 0; i < n_chunks; ++i) {
        const int s = i % n_stages;
        if (i >= n_stages && !tc::mbar_wait(&S.empty[s], ((i / n_stages) - 1) & 1, kWaitLimit)) {
          record_timeout(status);
          break;
        }
        const int tile0 = (c_begin + i) * kChunkTiles;
        const int nt = min(kChunkTiles, tile_end - tile0);
        const uint32_t bytes = static_cast<uint32_t>(nt * rec_bytes);
        tc::mbar_arrive_expect_tx(&S.full[s], bytes);
        tc::bulk_g2s(stages + s * stage_bytes, src + static_cast<size_t>(tile0) * rec_bytes, bytes, &S.full[s]);
      }
    }
  } else if (warp == kDecMmaWarp) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t id_s = tc::idesc_f16(128, 16, false), id_o = tc::idesc_f16(128, 16, true);
      const uint32_t bq = tc::smem_u32(sm + kBQOff), bp = tc::smem_u32(sm + kBPOff);
      const int ksteps = S.k_cols / 8;
      bool ok = true;
      for (int i = 0; i <= n_chunks && ok; ++i) {
        if (i < n_chunks) {
          const int bb = i & 1;
          if (!tc::mbar_wait(&S.kready[bb], (i >> 1) & 1, kWaitLimit)) { ok = false; break; }
          tc::fence_after_sync();
          for (int ks = 0; ks < ksteps; ++ks)
            tc::mma_ts(tbase + col_s(bb), tbase + col_ak(bb) + 8 * ks, tc::sdesc(bq + 512 * ks, 256, 128), id_s,
                       ks > 0);
          tc::mma_commit(&S.sfull[bb]);
        }
        if (i >= 1) {
          const int j = i - 1, bj = j & 1;
          if (!tc::mbar_wait(&S.pready[bj], (j >> 1) & 1, kWaitLimit) ||
              !tc::mbar_wait(&S.vready[bj], (j >> 1) & 1, kWaitLimit)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          for (int ks = 0; ks < kChunkTokens / 16; ++ks)
            tc::mma_ts(tbase + col_o(bj), tbase + col_av(bj) + 8 * ks,
                       tc::sdesc(bp + kBPBytes * bj + 512 * ks, 256, 128), id_o, ks > 0);
          tc::mma_commit(&S.ofull[bj]);
        }
      }
      if (!ok) record_timeout(status);
    }
  } else {
    // ---------------------------------------------------------------- compute warps
    const int wg = warp >> 2, qt = warp & 3;                // warp group, tensor-memory quarter
    const uint32_t lane_base = static_cast<uint32_t>(32 * qt) << 16;
    const uint32_t lane4 = static_cast<uint32_t>(lane) << 2;
    const int ngk = S.n_kgroups[wg];
    const uint32_t* kg = S.kgroup[wg];
    const int norm_off = 4 * kD * (bits_k + bits_v);
    const float qs0 = S.qscale[2 * wg], qs1 = S.qscale[2 * wg + 1];
    // Zero both K buffers once: columns past the last group stay zero (their Q' is 0 too).
    {
      uint32_t z[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) z[i] = 0u;
#pragma unroll
      for (int i = 0; i < 4; ++i) tc::tmem_st<16>(tbase + lane_base + 64 * wg + 16 * i, z);
    }
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f, o0 = 0.0f, o1 = 0.0f;
    float al00 = 0.0f, al01 = 0.0f, al10 = 0.0f, al11 = 0.0f;   // alpha[parity][query]
    float kn_prev = 0.0f, vn_prev = 0.0f;
    bool ok = true;

    auto softmax = [&](int j, float kn, float vn) {
      const int bj = j & 1;
      if (ok && !tc::mbar_wait(&S.sfull[bj], (j >> 1) & 1, kWaitLimit)) ok = false;
      tc::fence_after_sync();
      uint32_t sh[2], sl[2];
      tc::tmem_ld<2>(tbase + lane_base + col_s(bj) + 2 * wg, sh);
      tc::tmem_ld<2>(tbase + lane_base + col_s(bj) + 8 + 2 * wg, sl);
      tc::wait_ld();
      const int tile = (c_begin + j) * kChunkTiles + qt;
      const int tok = tile * kTile + lane;
      const bool valid = tile < tile_end && tok < seq_len;
      float s0 = (__uint_as_float(sh[0]) + __uint_as_float(sl[0])) * (kn * qs0);
      float s1 = (__uint_as_float(sh[1]) + __uint_as_float(sl[1])) * (kn * qs1);
      if (!valid) { s0 = -INFINITY; s1 = -INFINITY; }
      const int k0 = __reduce_max_sync(0xffffffffu, ordered(s0));
      const int k1 = __reduce_max_sync(0xffffffffu, ordered(s1));
      if (lane == 0) {
        S.xmax[bj][wg][qt][0] = from_ordered(k0);
        S.xmax[bj][wg][qt][1] = from_ordered(k1);
      }
      named_sync(1 + wg, 128);
      float c0 = S.xmax[bj][wg][0][0], c1 = S.xmax[bj][wg][0][1];
#pragma unroll
      for (int u = 1; u < 4; ++u) {
        c0 = fmaxf(c0, S.xmax[bj][wg][u][0]);
        c1 = fmaxf(c1, S.xmax[bj][wg][u][1]);
      }
      const float n0 = fmaxf(m0, c0), n1 = fmaxf(m1, c1);
      const float a0 = (m0 == -INFINITY) ? 0.0f : fast_exp2(m0 - n0);
      const float a1 = (m1 == -INFINITY) ? 0.0f : fast_exp2(m1 - n1);
      m0 = n0;
      m1 = n1;
      const float p0 = valid ? fast_exp2(s0 - n0) : 0.0f;
      const float p1 = valid ? fast_exp2(s1 - n1) : 0.0f;
      l0 = l0 * a0 + p0;
      l1 = l1 * a1 + p1;
      const float vs = valid ? vn * inv_sqrt_d : 0.0f;
      __half h0, lo0, h1, lo1;
      split_hilo(p0 * vs, h0, lo0);
      split_hilo(p1 * vs, h1, lo1);
      const int t = 32 * qt + lane;
      uint8_t* pb = sm + kBPOff + kBPBytes * bj + (t >> 3) * 256 + (t & 7) * 16 + 4 * wg;
      *reinterpret_cast<uint32_t*>(pb) = pack_half2(h0, h1);
      *reinterpret_cast<uint32_t*>(pb + 128) = pack_half2(lo0, lo1);
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&S.pready[bj]);
      if (bj) { al10 = a0; al11 = a1; } else { al00 = a0; al01 = a1; }
    };

    auto o_acc = [&](int j) {
      const int bj = j & 1;
      if (ok && !tc::mbar_wait(&S.ofull[bj], (j >> 1) & 1, kWaitLimit)) ok = false;
      tc::fence_after_sync();
      uint32_t oh[2], ol[2];
      tc::tmem_ld<2>(tbase + lane_base + col_o(bj) + 2 * wg, oh);
      tc::tmem_ld<2>(tbase + lane_base + col_o(bj) + 8 + 2 * wg, ol);
      tc::wait_ld();
      const float a0 = bj ? al10 : al00, a1 = bj ? al11 : al01;
      o0 = o0 * a0 + (__uint_as_float(oh[0]) + __uint_as_float(ol[0]));
      o1 = o1 * a1 + (__uint_as_float(oh[1]) + __uint_as_float(ol[1]));
    };

    for (int i = 0; i < n_chunks; ++i) {
      const int bb = i & 1, s = i % n_stages;
      if (ok && !tc::mbar_wait(&S.full[s], (i / n_stages) & 1, kWaitLimit)) ok = false;
      const uint8_t* st = stages + s * stage_bytes;
      // K-hat rows: token 32 qt + lane = token `lane` of tile qt.
      {
        const uint32_t* kw = reinterpret_cast<const uint32_t*>(st + qt * rec_bytes) + lane;
        const uint32_t ta = tbase + lane_base + col_ak(bb);
        for (int gi = 0; gi < ngk; ++gi) {
          const uint32_t g = kg[gi];
          k_group_any(static_cast<int>(g & 15u), kw, (g >> 4) & 0xfffu, ta + (g >> 16), sm, lane4);
        }
      }
      tc::wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&S.kready[bb]);
      if (i >= 2) o_acc(i - 2);          // also frees A_V, P' and O of this parity
      // V-hat^T rows: dim 32 qt + lane, tokens of tile wg -> columns 16 wg .. 16 wg + 15.
      {
        const uint32_t* vw = reinterpret_cast<const uint32_t*>(st + wg * rec_bytes + 4 * kD * bits_k) + 32 * qt + lane;
        v_tile_any(bits_v, vw, tbase + lane_base + col_av(bb) + 16 * wg, sm, lane4);
      }
      tc::wait_st();
      tc::fence_before_sync();
      const uint16_t* nrm = reinterpret_cast<const uint16_t*>(st + qt * rec_bytes + norm_off);
      const float kn = __half2float(__ushort_as_half(nrm[lane]));
      const float vn = __half2float(__ushort_as_half(nrm[kTile + lane]));
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(&S.vready[bb]);
        tc::mbar_arrive(&S.empty[s]);
      }
      if (i >= 1) softmax(i - 1, kn_prev, vn_prev);
      kn_prev = kn;
      vn_prev = vn;
    }
    if (n_chunks >= 1) softmax(n_chunks - 1, kn_prev, vn_prev);
    if (n_chunks >= 2) o_acc(n_chunks - 2);
    if (n_chunks >= 1) o_acc(n_chunks - 1);
    if (!ok) record_timeout(status);

    // ---------------------------------------------------------------- CTA result
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    if (lane == 0) {
      S.lpart[wg][qt][0] = l0;
      S.lpart[wg][qt][1] = l1;
    }
    named_sync(1 + wg, 128);
    const float L0 = S.lpart[wg][0][0] + S.lpart[wg][1][0] + S.lpart[wg][2][0] + S.lpart[wg][3][0];
    const float L1 = S.lpart[wg][0][1] + S.lpart[wg][1][1] + S.lpart[wg][2][1] + S.lpart[wg][3][1];
    const int d = 32 * qt + lane;
    const int h0 = 2 * wg, h1 = 2 * wg + 1;
    if (splits == 1) {
      float* ob = out + (static_cast<size_t>(b) * n_q_heads + hkv * G) * kD;
      if (h0 < G) ob[h0 * kD + d] = o0 / L0;
      if (h1 < G) ob[h1 * kD + d] = o1 / L1;
    } else {
      const size_t pb0 = (static_cast<size_t>(bh) * (splits + n_groups) + split) * 8;
      part_o[(pb0 + h0) * kD + d] = o0;
      part_o[(pb0 + h1) * kD + d] = o1;
      if (d == 0) {
        part_m[pb0 + h0] = m0;
        part_l[pb0 + h0] = L0;
        part_m[pb0 + h1] = m1;
        part_l[pb0 + h1] = L1;
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == kDecMmaWarp) tc::tmem_dealloc(tbase, kTmemCols);
  if (splits == 1) return;

  // ------------------------------------------------------------------ cross-split merge
  // Two levels: the last CTA of each group of kMergeGroup splits merges its group into a
  // group partial (entry splits + group); the last group merges the group partials.
  const int pitch = splits + n_groups;
  const int grp = split / kMergeGroup;
  const int g0 = grp * kMergeGroup, gn = min(splits, g0 + kMergeGroup) - g0;
  float* out_bh = out + (static_cast<size_t>(b) * n_q_heads + hkv * G) * kD;
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    unsigned* gt = tickets + gridDim.y + static_cast<size_t>(bh) * n_groups + grp;
    const unsigned t = atomicAdd(gt, 1u);
    S.last = (t == static_cast<unsigned>(gn - 1));
    if (S.last) *gt = 0u;
  }
  __syncthreads();
  if (!S.last) return;
  __threadfence();
  if (n_groups == 1) {
    merge_partials(S, stages, bh, pitch, 0, splits, part_m, part_l, part_o, 0, out_bh, G);
    return;
  }
  merge_partials(S, stages, bh, pitch, g0, gn, part_m, part_l, part_o, splits + grp, nullptr, G);
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned t = atomicAdd(&tickets[bh], 1u);
    S.last = (t == static_cast<unsigned>(n_groups - 1));
    if (S.last) tickets[bh] = 0u;
  }
  __syncthreads();
  if (!S.last) return;
  __threadfence();
  merge_partials(S, stages, bh, pitch, splits, n_groups, part_m, part_l, part_o, 0, out_bh, G);
}

}  // namespace kvq
