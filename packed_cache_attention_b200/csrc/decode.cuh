// Fused decode attention read straight from the packed Block-GTQ cache (page "RoPE-aware bit
// allocation for KV cache quantization", abstract: attention served from the packed cache;
// the NQKV review's editorial extensions propose folding the table lookup into attention).
//
// Grid: (splits, batch * n_kv_heads). Each CTA owns a contiguous range of 128-token chunks
// (4 tile records) of one (sequence, KV head) and walks it in segments of up to 16 chunks,
// each in two passes:
//   pass 1 (keys)   16 warps dequantize K codes through shared-memory lookup tables into
//                   tensor memory (K-hat rows, lane = token, one fp16 pair per column); one
//                   thread issues S^T[128 tokens][16] = Khat x Q'^T (tcgen05.mma, M 128, N 16,
//                   Q' hi rows 0-7 and lo rows 8-15 in shared memory); each thread keeps the
//                   scaled logits of its token in shared memory and a running maximum;
//   segment max     one exchange per warp group gives the segment's maximum per query row;
//                   the running (m, l, O) are rescaled once;
//   pass 2 (values) 16 warps dequantize V codes into V-hat^T rows (lane = dim); each thread
//                   turns its logits into P' = 2^(s - m) vnorm / sqrt(d), split into fp16 hi
//                   + lo (the B operand); O^T[128 dims][16] += Vhat^T x P'^T accumulates in
//                   tensor memory over the whole segment and is read once at its end.
// A load warp bulk-copies the key half (K words + norms) of every tile for pass 1 and the
// value half (norms + V words) for pass 2 through a ring of shared-memory stages. Q' carries
// f_b, log2(e)/sqrt(d) and a per-row power of two that keeps its fp16 split in range; the
// key norm scales S after the MMA. The K operand's columns come from the allocation's decode
// plan: width classes cut into groups of 4 block pairs (a class's last group 2 pairs when at
// most 2 remain), warp group g owning columns 24 g .. 24 g + 23; each thread decodes its
// groups into registers and writes them with one wide tensor-memory store per chunk. Warp
// group g handles query rows 2g, 2g+1 of the softmax and of O. Every hand-off is an mbarrier
// with a bounded wait.
// Splits write (m, l, O) partials to the workspace; the last CTA of a (sequence, KV head),
// found with an atomic ticket, merges them all and writes out = O / l.
#pragma once

#include "common.cuh"
#include "tcgen05.cuh"

namespace kvq {

constexpr int kDecComputeWarps = 16;
constexpr int kDecMmaWarp = 16;      // builds Q', issues the MMAs of even chunks
constexpr int kDecLoadWarp = 17;
constexpr int kDecMma2Warp = 18;     // issues the MMAs of odd chunks
constexpr int kDecThreads = 19 * 32;
constexpr int kChunkTiles = 4;
constexpr int kChunkTokens = kChunkTiles * kTile;   // = MMA M = tensor-memory lanes
constexpr int kSegChunks = 16;                       // chunks per two-pass segment
constexpr int kDecStagesMax = 8;
constexpr int kMaxMergeSplits = 160;
constexpr int kMergeGroup = 8;       // splits merged by the last CTA of each group (first level)
constexpr int kTargetCtas = 148;     // one CTA per SM on a 148-SM B200
constexpr int kGroupPairs = 4;       // block pairs (tensor-memory columns) per full K group
constexpr int kMaxKGroups = 16;      // per warp group (at most 24 groups per head in all)
constexpr int kMaxRuns = 8;          // runs of equal-width K groups per warp group
constexpr int kSlots = 6;            // K groups per warp group
constexpr int kSlotCols = 4 * kSlots;  // K columns per warp group
constexpr uint32_t kWaitLimit = 2000;   // suspended tries (about 2 s) before a wait gives up

// Tensor-memory columns (512 allocated).
constexpr uint32_t kTmemCols = 512;
// The key pass keeps 3 chunks in flight (its logits trail the dequantization by 2 chunks),
// the value pass 2.
__device__ __forceinline__ uint32_t col_ak(int b) { return 96u * b; }         // K-hat, 3 x 96
__device__ __forceinline__ uint32_t col_s(int b) { return 288u + 16u * b; }   // S, 3 x 16
__device__ __forceinline__ uint32_t col_av(int b) { return 336u + 64u * b; }  // V-hat^T, 2 x 64
__device__ __forceinline__ uint32_t col_o(int p) { return 464u + 16u * p; }  // O, 2 x 16 (chunk parity)

// Lookup-table image, built once per device (decode_lut_image) and bulk-copied into every
// CTA's shared memory at byte 0. Pair tables give the fp16 pair {c[i & m], c[i >> w]} for the
// 2w-bit index i of two consecutive codes: widths 1..3 keep one copy per lane (entry e of
// lane l at word 32 e + l) so that 32 lanes never share a bank; widths 4..6 keep one copy;
// widths 7, 8 use single-code fp16 tables.
__host__ __device__ constexpr int lut_off(int w) {
  return w == 1 ? 0 : w == 2 ? 512 : w == 3 ? 2560 : w == 4 ? 10752 : w == 5 ? 11776 : w == 6 ? 15872
                                                                                       : w == 7 ? 32256 : 32512;
}
constexpr int kLutBytes = 33024;
// Shared-memory map (byte offsets from the start of dynamic shared memory).
constexpr int kAllocOff = kLutBytes;                 // copy of the KV head's kvq_head_alloc
constexpr int kBQOff = ((kAllocOff + static_cast<int>(sizeof(kvq_head_alloc)) + 127) / 128) * 128;
                                                     // Q' (B operand of S), K-major, <= 256 K elements
constexpr int kBQBytes = 32 * 256;
constexpr int kBPOff = kBQOff + kBQBytes;            // P' (B operand of O), 2 buffers, N-major
constexpr int kBPBytes = 4096;
constexpr int kStashOff = kBPOff + 2 * kBPBytes;     // logits of a segment: [chunk][row][token] fp32
constexpr int kStashBytes = kSegChunks * 8 * kChunkTokens * 4;
constexpr int kHdrOff = kStashOff + kStashBytes;
static_assert(kLutBytes % 16 == 0 && kAllocOff % 16 == 0 && sizeof(kvq_head_alloc) % 16 == 0,
              "bulk-copied regions must be 16-byte multiples");
static_assert(kBQOff >= kAllocOff + static_cast<int>(sizeof(kvq_head_alloc)) && kBQOff % 128 == 0,
              "Q' must not overlap the allocation copy");

struct DecHeader {
  uint64_t full[kDecStagesMax];
  uint64_t empty[kDecStagesMax];
  uint64_t kready[3], sfull[3], vpready[2], ofull[2];
  uint64_t setup;                    // lookup tables + allocation record copied in
  uint64_t qready;                   // Q' and qscale written (MMA warp)
  uint32_t tmem_base;
  float qscale[8];                   // 2^e that undoes the range scaling of Q' row h
  float xmax[2][4][4][2];            // segment max: [segment parity][warp group][quarter][row]
  float lpart[4][4][2];              // row sums: [warp group][quarter][row]
  int last;
  float mw[8][kMaxMergeSplits];      // cross-split merge: member m, then weight 2^(m_s - M)
  float ml[8][kMaxMergeSplits];      // cross-split merge: member l
  float Lsum[8];
  float Mmax[8];
};

__host__ __device__ constexpr int decode_stage_off() {
  return kHdrOff + ((static_cast<int>(sizeof(DecHeader)) + 127) / 128) * 128;
}

// Byte sizes of the key half (K words + K norms) and the value half (V norms + V words) of a
// tile record. A stage holds 4 tiles; a tile's slot also covers K word rows 4 bits_k and
// 4 bits_k + 1 (up to byte 512 bits_k + 256), which the last K groups of a token read past
// the end of its stream, so every read stays inside the slot.
__host__ __device__ constexpr int key_half_bytes(int bits_k) { return 4 * kD * bits_k + 2 * kTile; }
__host__ __device__ constexpr int value_half_bytes(int bits_v) { return 2 * kTile + 4 * kD * bits_v; }
__host__ __device__ constexpr int stage_tile_stride(int bits_k, int bits_v) {
  return (4 * kD * bits_k + 256) > value_half_bytes(bits_v) ? (4 * kD * bits_k + 256) : value_half_bytes(bits_v);
}

// Host: the lookup-table image from the fp16 centroid table (width w at c16 + 2^w - 2).
inline void decode_lut_image(const uint16_t* c16, uint8_t* img) {
  for (int w = 1; w <= 6; ++w) {
    const uint16_t* c = c16 + (1 << w) - 2;
    uint32_t* t = reinterpret_cast<uint32_t*>(img + lut_off(w));
    const int copies = (w <= 3) ? 32 : 1;
    for (int e = 0; e < (1 << (2 * w)); ++e)
      for (int l = 0; l < copies; ++l)
        t[e * copies + l] = static_cast<uint32_t>(c[e & ((1 << w) - 1)]) | (static_cast<uint32_t>(c[e >> w]) << 16);
  }
  for (int w = 7; w <= 8; ++w) {
    uint16_t* t = reinterpret_cast<uint16_t*>(img + lut_off(w));
    for (int e = 0; e < (1 << w); ++e) t[e] = c16[(1 << w) - 2 + e];
  }
}

// Device copy of the image (single translation unit; uploaded once per device).
__device__ __align__(16) uint8_t g_dec_lut[kLutBytes];

// ---------------------------------------------------------------- code extraction + lookup

// Bits [p, p + n) of the 64-bit value hi:lo (p, n constant after unrolling, n <= 16).
__device__ __forceinline__ uint32_t field(uint32_t lo, uint32_t hi, int p, int n) {
  uint32_t v;
  if (p >= 32) v = hi >> (p - 32);
  else if (p + n <= 32) v = lo >> p;
  else v = __funnelshift_r(lo, hi, p);
  return v & ((1u << n) - 1u);
}

// Bits [p, p + n) of hi:lo moved to bit position `sh` (p, n, sh constant after unrolling):
// one funnel shift (or plain shift) and one mask.
__device__ __forceinline__ uint32_t field_at(uint32_t lo, uint32_t hi, int p, int n, int sh) {
  const uint32_t m = ((1u << n) - 1u) << sh;
  uint32_t v;
  if (p >= sh) {
    const int q = p - sh;
    v = (q >= 32) ? (hi >> (q - 32)) : (q + sh + n <= 32 ? (lo >> q) : __funnelshift_r(lo, hi, q));
  } else {
    v = lo << (sh - p);
  }
  return v & m;
}

// fp16 pair for two consecutive codes: code_a = bits [p, p + W), code_b = bits [p + W, p + 2W)
// of hi:lo; code_a goes to the low half. The pair index lands directly at its table offset
// (x 128 bytes plus the lane's word for the per-lane copies, x 4 bytes otherwise).
template <int W>
__device__ __forceinline__ uint32_t pair_value(uint32_t lo, uint32_t hi, int p, const uint8_t* sm, uint32_t lane4) {
  if constexpr (W <= 3) {
    return *reinterpret_cast<const uint32_t*>(sm + lut_off(W) + (field_at(lo, hi, p, 2 * W, 7) | lane4));
  } else if constexpr (W <= 6) {
    return *reinterpret_cast<const uint32_t*>(sm + lut_off(W) + field_at(lo, hi, p, 2 * W, 2));
  } else {
    const uint8_t* t = sm + lut_off(W);
    return static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(t + field_at(lo, hi, p, W, 1))) |
           (static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(t + field_at(lo, hi, p + W, W, 1))) << 16);
  }
}

// Values of NP consecutive block pairs of width W whose first code starts at bit `off` of
// this lane's token stream; kw points at word 0 of the token (word i at kw[32 i]).
template <int W, int NP>
__device__ __forceinline__ void k_group_vals(const uint32_t* kw, uint32_t off, const uint8_t* sm, uint32_t lane4,
                                             uint32_t (&v)[NP]) {
  const uint32_t j0 = off >> 5, s = off & 31u;
  const uint32_t x0 = kw[j0 * 32], x1 = kw[(j0 + 1) * 32];
  const uint32_t x2 = (2 * W * NP > 32) ? kw[(j0 + 2) * 32] : 0u;
  const uint32_t r0 = __funnelshift_r(x0, x1, s);
  const uint32_t r1 = __funnelshift_r(x1, x2, s);
#pragma unroll
  for (int k = 0; k < NP; ++k) v[k] = pair_value<W>(r0, r1, 2 * W * k, sm, lane4);
}

// Values of the K group in one register slot: e = width | bit offset << 8 (width 0: an empty
// slot, left zero). A group with only 2 real pairs is decoded as 4; the other 2 columns have
// a zero Q' row. Slots sit at compile-time register positions and reach tensor memory in one
// wide store per chunk afterwards: small stores issued between the lookups were measured to
// slow the whole dequantization several times over.
__device__ __forceinline__ void k_slot(uint32_t e, const uint32_t* kw, const uint8_t* sm, uint32_t lane4,
                                       uint32_t (&t)[kGroupPairs]) {
  const uint32_t off = e >> 8;
  switch (e & 15u) {
    case 1: k_group_vals<1, kGroupPairs>(kw, off, sm, lane4, t); break;
    case 2: k_group_vals<2, kGroupPairs>(kw, off, sm, lane4, t); break;
    case 3: k_group_vals<3, kGroupPairs>(kw, off, sm, lane4, t); break;
    case 4: k_group_vals<4, kGroupPairs>(kw, off, sm, lane4, t); break;
    case 5: k_group_vals<5, kGroupPairs>(kw, off, sm, lane4, t); break;
    case 6: k_group_vals<6, kGroupPairs>(kw, off, sm, lane4, t); break;
    case 7: k_group_vals<7, kGroupPairs>(kw, off, sm, lane4, t); break;
    case 8: k_group_vals<8, kGroupPairs>(kw, off, sm, lane4, t); break;
    default: t[0] = 0u; t[1] = 0u; t[2] = 0u; t[3] = 0u; break;
  }
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
    v[u] = pair_value<BV>(x[p >> 5], x[(p >> 5) + 1], p & 31, sm, lane4);
  }
  tc::tmem_st<16>(taddr, v);
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

// Merge the n (m, l, O) partials of (sequence, KV head) bh (entries 0..n-1 of its row of the
// workspace) into out = O / l for its G real query heads. Called by every thread of the CTA:
// all members' (m, l) are fetched in one round, then 512 threads sum O (256 float4 quads,
// two halves of the member list each, 8 loads in flight).
__device__ __forceinline__ void merge_partials(DecHeader& S, uint8_t* scratch, int bh, int pitch, int n,
                                               const float* part_m, const float* part_l, const float* part_o,
                                               float* out, int G) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t row = static_cast<size_t>(bh) * pitch * 8;
  for (int i = tid; i < 8 * n; i += blockDim.x) {
    const int s = i >> 3, hg = i & 7;
    S.mw[hg][s] = __ldcg(part_m + row + i);
    S.ml[hg][s] = __ldcg(part_l + row + i);
  }
  __syncthreads();
  if (warp < 8) {
    const int hg = warp;
    float M = -INFINITY;
    for (int s = lane; s < n; s += 32) M = fmaxf(M, S.mw[hg][s]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.0f;
    for (int s = lane; s < n; s += 32) {
      const float ms = S.mw[hg][s];
      const float wt = (ms == -INFINITY) ? 0.0f : fast_exp2(ms - M);
      S.mw[hg][s] = wt;
      L += S.ml[hg][s] * wt;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (lane == 0) S.Lsum[hg] = L;
  }
  __syncthreads();
  const int quad = tid & 255, half = tid >> 8;
  const int hg = quad >> 5, j4 = quad & 31;
  const int s_mid = n / 2;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  if (half < 2) {
    const int s0 = half ? s_mid : 0, s1 = half ? n : s_mid;
    const float4* po = reinterpret_cast<const float4*>(part_o) + (row + hg) * (kD / 4) + j4;
#pragma unroll 8
    for (int s = s0; s < s1; ++s) {
      const float wt = S.mw[hg][s];
      const float4 v = __ldcg(po + static_cast<size_t>(s) * 8 * (kD / 4));
      o.x += v.x * wt; o.y += v.y * wt; o.z += v.z * wt; o.w += v.w * wt;
    }
  }
  float4* red = reinterpret_cast<float4*>(scratch);
  if (half == 1) red[quad] = o;
  __syncthreads();
  if (half == 0 && hg < G) {
    const float4 v = red[quad];
    const float inv = 1.0f / S.Lsum[hg];
    reinterpret_cast<float4*>(out + static_cast<size_t>(hg) * kD)[j4] =
        make_float4((o.x + v.x) * inv, (o.y + v.y) * inv, (o.z + v.z) * inv, (o.w + v.w) * inv);
  }
}

// ---------------------------------------------------------------- the kernel

// One instantiation per value width BVT (= bits_v).
template <int DT, int BVT>
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
  const int n_segs = (n_chunks + kSegChunks - 1) / kSegChunks;
  const int tile_end = min(n_tiles, c_end * kChunkTiles);
  const uint8_t* src = packed + static_cast<size_t>(bh) * tiles_cap * rec_bytes;
  const int khalf = key_half_bytes(bits_k), vhalf = value_half_bytes(bits_v);
  const int tstride = stage_tile_stride(bits_k, bits_v);
  const int stage_bytes = kChunkTiles * tstride;
  const float inv_sqrt_d = 0.08838834764831845f;
  constexpr int kSetupThreads = (kDecComputeWarps + 2) * 32;   // compute warps and both MMA warps

  // ------------------------------------------------------------------ barriers
  if (tid == 0) {
    for (int i = 0; i < kDecStagesMax; ++i) {
      tc::mbar_init(&S.full[i], 1);
      tc::mbar_init(&S.empty[i], kDecComputeWarps);
    }
    for (int i = 0; i < 3; ++i) {
      tc::mbar_init(&S.kready[i], kDecComputeWarps);
      tc::mbar_init(&S.sfull[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&S.vpready[i], kDecComputeWarps);
      tc::mbar_init(&S.ofull[i], 1);
    }
    tc::mbar_init(&S.setup, 1);
    tc::mbar_init(&S.qready, 1);
    tc::mbar_fence_init();
  }
  __syncthreads();

  if (warp == kDecLoadWarp) {
    // ---------------------------------------------------------------- bulk loads
    // Items in consumption order: per segment the key halves of its chunks, then the value
    // halves; item k uses stage k % n_stages.
    if (lane == 0) {
      tc::mbar_arrive_expect_tx(&S.setup, kLutBytes + static_cast<uint32_t>(sizeof(kvq_head_alloc)));
      tc::bulk_g2s(sm, g_dec_lut, kLutBytes, &S.setup);
      tc::bulk_g2s(sm + kAllocOff, al, sizeof(kvq_head_alloc), &S.setup);
      int k = 0;
      bool ok = true;
      for (int sg = 0; sg < n_segs && ok; ++sg) {
        const int u0 = sg * kSegChunks, nu = min(kSegChunks, n_chunks - u0);
        for (int half = 0; half < 2 && ok; ++half) {
          const int bytes = half ? vhalf : khalf, off = half ? khalf : 0;
          for (int u = 0; u < nu; ++u, ++k) {
            const int s = k % n_stages;
            if (k >= n_stages && !tc::mbar_wait(&S.empty[s], ((k / n_stages) - 1) & 1, kWaitLimit)) {
              ok = false;
              break;
            }
            const int tile0 = (c_begin + u0 + u) * kChunkTiles;
            const int nt = min(kChunkTiles, tile_end - tile0);
            tc::mbar_arrive_expect_tx(&S.full[s], static_cast<uint32_t>(nt * bytes));
            for (int t = 0; t < nt; ++t)
              tc::bulk_g2s(stages + s * stage_bytes + t * tstride,
                           src + static_cast<size_t>(tile0 + t) * rec_bytes + off, static_cast<uint32_t>(bytes),
                           &S.full[s]);
          }
        }
      }
      if (!ok) record_timeout(status);
    }
  } else {
    // ---------------------------------------------------------------- setup (warps 0..16)
    // The compute warps start on the first chunk as soon as the tables and the allocation
    // record (which carries the K group plan) are in; the MMA warp meanwhile builds Q'.
    if (warp == kDecMmaWarp) tc::tmem_alloc(&S.tmem_base, kTmemCols);
    tc::fence_before_sync();
    named_sync(5, kSetupThreads);
    tc::fence_after_sync();
    const uint32_t tbase = S.tmem_base;
    if (!tc::mbar_wait(&S.setup, 0, kWaitLimit)) record_timeout(status);
    const kvq_head_alloc& A = *reinterpret_cast<const kvq_head_alloc*>(sm + kAllocOff);

    if (warp == kDecMmaWarp || warp == kDecMma2Warp) {
      const int par = (warp == kDecMmaWarp) ? 0 : 1;   // chunk parity this warp issues for
      const int k_cols = 4 * kSlotCols;
      if (par == 0) {
      // -------------------------------------------------------------- Q' (whole warp)
      // Row h: q_h * f_b * log2(e) / sqrt(d), scaled by 2^-e so that its largest |value| is in
      // [0.5, 1); qscale[h] = 2^e multiplies the product back. B operand of S, K-major, no
      // swizzle: element (n, k) at (k/8)*256 + (n/8)*128 + (n%8)*16 + (k%8)*2; K element
      // k = 2c + r is dim b + 64 r of the block in column c; n < 8: hi part of row n, n >= 8:
      // lo part of row n - 8.
      float* qtmp = reinterpret_cast<float*>(sm + kBPOff);   // [8][128] fp32 until P' is first written
      float qv[8][4];
#pragma unroll
      for (int hg = 0; hg < 8; ++hg)
#pragma unroll
        for (int u = 0; u < 4; ++u)
          qv[hg][u] = (hg < G) ? Elem<DT>::to_f32(q[b * qsb + (hkv * G + hg) * qsh + lane + 32 * u]) : 0.0f;
#pragma unroll
      for (int hg = 0; hg < 8; ++hg) {
        float mx = 0.0f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = lane + 32 * u;
          qv[hg][u] *= A.dequant[j % kH] * (inv_sqrt_d * kLog2e);
          mx = fmaxf(mx, fabsf(qv[hg][u]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        int e = 0;
        if (mx > 0.0f) frexpf(mx, &e);
        if (lane == 0) S.qscale[hg] = ldexpf(1.0f, e);
        const float sc = ldexpf(1.0f, -e);
#pragma unroll
        for (int u = 0; u < 4; ++u) qtmp[hg * kD + lane + 32 * u] = qv[hg][u] * sc;
      }
      __syncwarp();
      const int k_elems = 2 * k_cols;
      for (int i = lane; i < 8 * k_elems; i += 32) {
        const int n = i / k_elems, k = i - n * k_elems;
        const int blk = A.plan_col_block[k >> 1];
        __half hi = __float2half_rn(0.0f), lo = hi;
        if (blk >= 0) split_hilo(qtmp[n * kD + blk + kH * (k & 1)], hi, lo);
        const int base = (k >> 3) * 256 + (k & 7) * 2;
        *reinterpret_cast<__half*>(sm + kBQOff + base + n * 16) = hi;
        *reinterpret_cast<__half*>(sm + kBQOff + base + 128 + n * 16) = lo;
      }
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&S.qready);
      }
      // -------------------------------------------------------------- MMA issue
      // Two issuing threads, one per chunk parity: independent MMA chains overlap in the
      // tensor pipe, whose cost per instruction is mostly latency at these small tiles.
      if (lane == 0) {
        if (par == 1 && !tc::mbar_wait(&S.qready, 0, kWaitLimit)) record_timeout(status);
        const uint32_t id_s = tc::idesc_f16(128, 16, false), id_o = tc::idesc_f16(128, 16, true);
        const uint32_t bq = tc::smem_u32(sm + kBQOff), bp = tc::smem_u32(sm + kBPOff);
        // k-steps (8 columns each) that hold at least one real block pair
        uint32_t kmask = 0u;
        for (int c = 0; c < k_cols; ++c)
          if (A.plan_col_block[c] >= 0) kmask |= 1u << (c >> 3);
        const int first_ks = __ffs(kmask) - 1;
        // Every k-step's B descriptor, built once (the 14-bit start field wraps, so offsets are
        // not added to a built descriptor).
        uint64_t dq[12], dpv[2][kChunkTokens / 16];
#pragma unroll
        for (int ks = 0; ks < 12; ++ks) dq[ks] = tc::sdesc(bq + 512 * ks, 256, 128);
#pragma unroll
        for (int bb = 0; bb < 2; ++bb)
#pragma unroll
          for (int ks = 0; ks < kChunkTokens / 16; ++ks)
            dpv[bb][ks] = (bb == par) ? tc::sdesc(bp + kBPBytes * bb + 512 * ks, 256, 128) : 0ull;
        int kc = 0, vc = 0;
        bool ok = true;
        for (int sg = 0; sg < n_segs && ok; ++sg) {
          const int nu = min(kSegChunks, n_chunks - sg * kSegChunks);
          for (int u = 0; u < nu; ++u, ++kc) {
            if ((kc & 1) != par) continue;
            const int bb = kc % 3;
            if (!tc::mbar_wait(&S.kready[bb], (kc / 3) & 1, kWaitLimit)) { ok = false; break; }
            tc::fence_after_sync();
            const uint32_t d = tbase + col_s(bb), a = tbase + col_ak(bb);
#pragma unroll
            for (int ks = 0; ks < 12; ++ks)
              if (kmask & (1u << ks)) tc::mma_ts(d, a + 8 * ks, dq[ks], id_s, ks != first_ks);
            tc::mma_commit(&S.sfull[bb]);
          }
          for (int u = 0; u < nu && ok; ++u, ++vc) {
            if ((vc & 1) != par) continue;
            const int bb = vc & 1;
            if (!tc::mbar_wait(&S.vpready[bb], (vc >> 1) & 1, kWaitLimit)) { ok = false; break; }
            tc::fence_after_sync();
            const uint32_t a = tbase + col_av(bb), d = tbase + col_o(bb);
            tc::mma_ts(d, a, dpv[par][0], id_o, u >= 2);   // first chunk of this parity starts O
#pragma unroll
            for (int ks = 1; ks < kChunkTokens / 16; ++ks) tc::mma_ts(d, a + 8 * ks, dpv[par][ks], id_o, 1u);
            tc::mma_commit(&S.ofull[bb]);
          }
        }
        if (!ok) record_timeout(status);
      }
    } else {
      // -------------------------------------------------------------- compute warps
      const int wg = warp >> 2, qt = warp & 3;                // warp group, tensor-memory quarter
      const uint32_t lane_base = static_cast<uint32_t>(32 * qt) << 16;
      const uint32_t lane4 = static_cast<uint32_t>(lane) << 2;
      const int t_lane = 32 * qt + lane;                      // token of a chunk (pass 1), dim (pass 2)
      // This warp group's K slots: slot i = plan entry i, as width | bit offset << 8 (0 = empty).
      uint32_t slot_e[kSlots];
      {
        uint32_t mine = 0u;
        const int n_runs = min(max(A.plan_n_runs[wg], 0), kMaxRuns);
        if (lane < kSlots)
          for (int r = 0; r < n_runs; ++r) {
            const uint32_t e = A.plan_run[wg][r];
            const int first = (e >> 8) & 0xff, n = (e >> 16) & 0xff;
            if (lane >= first && lane < first + n) mine = (e & 15u) | ((A.plan_group[wg][lane] & 0xffffu) << 8);
          }
#pragma unroll
        for (int i = 0; i < kSlots; ++i) slot_e[i] = __shfl_sync(0xffffffffu, mine, i);
      }
      float qs0 = 1.0f, qs1 = 1.0f;
      bool have_q = false;
      float* stash = reinterpret_cast<float*>(sm + kStashOff);
      // Zero both K buffers once: columns past the last group stay zero (their Q' is 0 too).
      {
        uint32_t z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = 0u;
#pragma unroll
        for (int i = 0; i < 4; ++i) tc::tmem_st<16>(tbase + lane_base + 64 * wg + 16 * i, z);
      }
      float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f, o0 = 0.0f, o1 = 0.0f;
      int k = 0, kc0 = 0, vc0 = 0;
      bool ok = true;

      // Logits of chunk u of the segment (K count j): s = S * knorm * qscale, -inf past the end.
      auto logits = [&](int u0, int u, int j, float kn, float& sm0, float& sm1) {
        const int bj = j % 3;
        if (!have_q) {   // Q' scaling of this warp group's rows (written by the MMA warp)
          if (ok && !tc::mbar_wait(&S.qready, 0, kWaitLimit)) ok = false;
          qs0 = S.qscale[2 * wg];
          qs1 = S.qscale[2 * wg + 1];
          have_q = true;
        }
        if (ok && !tc::mbar_wait(&S.sfull[bj], (j / 3) & 1, kWaitLimit)) ok = false;
        tc::fence_after_sync();
        uint32_t sh[2], sl[2];
        tc::tmem_ld2x2_wait(tbase + lane_base + col_s(bj) + 2 * wg, tbase + lane_base + col_s(bj) + 8 + 2 * wg, sh, sl);
        const int tile = (c_begin + u0 + u) * kChunkTiles + qt;
        const bool valid = tile < tile_end && tile * kTile + lane < seq_len;
        float s0 = (__uint_as_float(sh[0]) + __uint_as_float(sl[0])) * (kn * qs0);
        float s1 = (__uint_as_float(sh[1]) + __uint_as_float(sl[1])) * (kn * qs1);
        if (!valid) { s0 = -INFINITY; s1 = -INFINITY; }
        stash[(u * 8 + 2 * wg) * kChunkTokens + t_lane] = s0;
        stash[(u * 8 + 2 * wg + 1) * kChunkTokens + t_lane] = s1;
        sm0 = fmaxf(sm0, s0);
        sm1 = fmaxf(sm1, s1);
      };

      for (int sg = 0; sg < n_segs; ++sg) {
        const int u0 = sg * kSegChunks, nu = min(kSegChunks, n_chunks - u0);
        // ------------------------------------------------------------ pass 1: keys
        float sm0 = -INFINITY, sm1 = -INFINITY, kn1 = 0.0f, kn2 = 0.0f;   // norms of chunks u-1, u-2
        for (int u = 0; u < nu; ++u, ++k) {
          const int s = k % n_stages, j = kc0 + u;
          if (ok && !tc::mbar_wait(&S.full[s], (k / n_stages) & 1, kWaitLimit)) ok = false;
          const uint8_t* st = stages + s * stage_bytes + qt * tstride;   // tile qt: token `lane`
          const uint32_t* kw = reinterpret_cast<const uint32_t*>(st) + lane;
          const uint32_t ta = tbase + lane_base + col_ak(j % 3) + kSlotCols * wg;
          {
            uint32_t t[kSlots][kGroupPairs];
#pragma unroll
            for (int i = 0; i < kSlots; ++i) k_slot(slot_e[i], kw, sm, lane4, t[i]);
            uint32_t v16[16], v8[8];
#pragma unroll
            for (int i = 0; i < 16; ++i) v16[i] = t[i / 4][i % 4];
#pragma unroll
            for (int i = 0; i < 8; ++i) v8[i] = t[4 + i / 4][i % 4];
            tc::tmem_st<16>(ta, v16);
            tc::tmem_st<8>(ta + 16, v8);
          }
          const float kn = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(st + 4 * kD * bits_k)[lane]));
          tc::wait_st();
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) {
            tc::mbar_arrive(&S.kready[j % 3]);
            tc::mbar_arrive(&S.empty[s]);
          }
          if (u >= 2) logits(u0, u - 2, j - 2, kn2, sm0, sm1);
          kn2 = kn1;
          kn1 = kn;
        }
        if (nu >= 2) logits(u0, nu - 2, kc0 + nu - 2, kn2, sm0, sm1);
        logits(u0, nu - 1, kc0 + nu - 1, kn1, sm0, sm1);
        kc0 += nu;
        // ------------------------------------------------------------ segment maximum
        {
          const int k0 = __reduce_max_sync(0xffffffffu, ordered(sm0));
          const int k1 = __reduce_max_sync(0xffffffffu, ordered(sm1));
          if (lane == 0) {
            S.xmax[sg & 1][wg][qt][0] = from_ordered(k0);
            S.xmax[sg & 1][wg][qt][1] = from_ordered(k1);
          }
          named_sync(1 + wg, 128);
          float c0 = S.xmax[sg & 1][wg][0][0], c1 = S.xmax[sg & 1][wg][0][1];
#pragma unroll
          for (int v = 1; v < 4; ++v) {
            c0 = fmaxf(c0, S.xmax[sg & 1][wg][v][0]);
            c1 = fmaxf(c1, S.xmax[sg & 1][wg][v][1]);
          }
          const float n0 = fmaxf(m0, c0), n1 = fmaxf(m1, c1);
          const float a0 = (m0 == -INFINITY) ? 0.0f : fast_exp2(m0 - n0);
          const float a1 = (m1 == -INFINITY) ? 0.0f : fast_exp2(m1 - n1);
          m0 = n0;
          m1 = n1;
          l0 *= a0; l1 *= a1;
          o0 *= a0; o1 *= a1;
        }
        // ------------------------------------------------------------ pass 2: values
        for (int u = 0; u < nu; ++u, ++k) {
          const int s = k % n_stages, j = vc0 + u, bj = j & 1;
          if (ok && !tc::mbar_wait(&S.full[s], (k / n_stages) & 1, kWaitLimit)) ok = false;
          if (j >= 2 && ok && !tc::mbar_wait(&S.ofull[bj], ((j - 2) >> 1) & 1, kWaitLimit)) ok = false;
          const uint8_t* st = stages + s * stage_bytes;
          // V-hat^T row: dim t_lane, tokens of tile wg -> columns 16 wg .. 16 wg + 15.
          const uint32_t* vw = reinterpret_cast<const uint32_t*>(st + wg * tstride + 2 * kTile) + t_lane;
          v_tile<BVT>(vw, tbase + lane_base + col_av(bj) + 16 * wg, sm, lane4);
          // P' of token t_lane (tile qt, token lane), rows 2 wg, 2 wg + 1.
          const float vn = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(st + qt * tstride)[lane]));
          const float s0 = stash[(u * 8 + 2 * wg) * kChunkTokens + t_lane];
          const float s1 = stash[(u * 8 + 2 * wg + 1) * kChunkTokens + t_lane];
          const bool valid = s0 != -INFINITY;
          const float p0 = valid ? fast_exp2(s0 - m0) : 0.0f;
          const float p1 = valid ? fast_exp2(s1 - m1) : 0.0f;
          l0 += p0;
          l1 += p1;
          const float vs = valid ? vn * inv_sqrt_d : 0.0f;
          __half h0, lo0, h1, lo1;
          split_hilo(p0 * vs, h0, lo0);
          split_hilo(p1 * vs, h1, lo1);
          uint8_t* pb = sm + kBPOff + kBPBytes * bj + (t_lane >> 3) * 256 + (t_lane & 7) * 16 + 4 * wg;
          *reinterpret_cast<uint32_t*>(pb) = pack_half2(h0, h1);
          *reinterpret_cast<uint32_t*>(pb + 128) = pack_half2(lo0, lo1);
          tc::wait_st();
          tc::fence_proxy_async_smem();
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) {
            tc::mbar_arrive(&S.vpready[bj]);
            tc::mbar_arrive(&S.empty[s]);
          }
        }
        vc0 += nu;
        // ------------------------------------------------------------ segment O
        // One accumulator per chunk parity: wait for the last chunk of each, add both.
        {
          const int jl = vc0 - 1;
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int jq = jl - q;
            if (q == 1 && nu < 2) break;
            if (ok && !tc::mbar_wait(&S.ofull[jq & 1], (jq >> 1) & 1, kWaitLimit)) ok = false;
            tc::fence_after_sync();
            uint32_t oh[2], ol[2];
            tc::tmem_ld2x2_wait(tbase + lane_base + col_o(jq & 1) + 2 * wg, tbase + lane_base + col_o(jq & 1) + 8 + 2 * wg,
                                oh, ol);
            o0 += __uint_as_float(oh[0]) + __uint_as_float(ol[0]);
            o1 += __uint_as_float(oh[1]) + __uint_as_float(ol[1]);
          }
          tc::fence_before_sync();
        }
      }
      if (!ok) record_timeout(status);

      // -------------------------------------------------------------- CTA result
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
      const int d = t_lane;
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
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == kDecMmaWarp) tc::tmem_dealloc(S.tmem_base, kTmemCols);
  if (splits == 1) return;

  // ------------------------------------------------------------------ cross-split merge
  // The last CTA of this (sequence, KV head), found with an atomic ticket, merges all splits.
  const int pitch = splits + n_groups;
  float* out_bh = out + (static_cast<size_t>(b) * n_q_heads + hkv * G) * kD;
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned t = atomicAdd(&tickets[bh], 1u);
    S.last = (t == static_cast<unsigned>(splits - 1));
    if (S.last) tickets[bh] = 0u;
  }
  __syncthreads();
  if (!S.last) return;
  __threadfence();
  merge_partials(S, stages, bh, pitch, splits, part_m, part_l, part_o, out_bh, G);
}

}  // namespace kvq
