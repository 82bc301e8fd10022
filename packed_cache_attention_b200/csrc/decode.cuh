// Fused decode attention read straight from the packed Block-GTQ cache (page "RoPE-aware bit
// allocation for KV cache quantization", abstract: attention served from the packed cache;
// the NQKV review's editorial extensions propose folding the table lookup into attention).
//
// Grid: (splits, batch * n_kv_heads); 4 warps per CTA; each CTA owns a contiguous range of
// 32-token tiles of one (sequence, KV head) and each warp every 4th tile of that range.
// Tiles are staged into shared memory with 16-byte cp.async copies, kStages deep per warp.
//
// Per tile, on the tensor cores (mma.sync, fp16 operands, fp32 accumulate), for the G <= 8
// query heads of the KV head held as 16 rows (8 heads' fp16 high parts, 8 low parts):
//   S^T[16][32 tokens] = Q'[16][k-steps of 4 RoPE blocks] x Khat_codes^T
//     Q'_{h,j} = q_{h,j} f_b log2(e) / sqrt(d) scaled per head by a power of two; the key
//     norm is applied to S after the MMA, so the B operand is the raw fp16 centroid.
//   online softmax in the log2 domain, P' = p * vnorm / sqrt(d) split into fp16 hi + lo,
//   O[16][128] += P'[16][32 tokens] x Vhat_codes[32][128].
// Fragment order follows the tile layout: lane (g = lane/4, c = lane%4) holds token g + 8j
// (n-tile j) for K and tokens 8(m/2) + 2c + (m%2) for V, so its codes are the nibbles at
// bits (g%4) + 4m of a K word and c + 4m of a V word.
// Splits write (m, l, O) partials to the workspace; the last CTA of a (sequence, KV head),
// found with an atomic ticket, merges them in split order and writes out = O / l.
#pragma once

#include "common.cuh"

namespace kvq {

constexpr int kDecWarps = 16;
constexpr int kDecStages = 3;        // deepest cp.async pipeline per warp (fewer when records are large)
constexpr int kMaxSteps = 32;
constexpr int kMaxMergeSplits = 160;
constexpr int kMergeGroup = 8;      // splits merged by the last CTA of each group (first level)
constexpr int kTargetCtas = 148;   // 1 CTA of 16 warps per SM on a 148-SM B200

struct DecodeSmem {
  uint4 kstep[kMaxSteps][8][4];     // per k-step, head row g, lane c: {Q' hi, Q' lo, K word offset + H, 0}
  float qp[8][kD];                  // Q' in fp32 before scaling
  float qmul[8];                    // 2^e that undoes the per-head scaling of Q'
  uint16_t cent[kCentroidCount];    // fp16 centroid bit patterns
  uint4 lut8[4];                    // widths 1..3: {lo bytes 0-3, lo 4-7, hi 0-3, hi 4-7}
  uint4 lut16[2];                   // width 4: {loA0, loA1, loB0, loB1}, {hiA0, hiA1, hiB0, hiB1}
  uint16_t woff[kH];
  int8_t step_blk[kMaxSteps][4];
  uint8_t step_w[kMaxSteps];
  int cls_w[9];                      // k-steps grouped by width: width of class i,
  int cls_begin[10];                 // first step of class i (cls_begin[n_cls] = n_steps)
  int n_cls;
  int n_steps;
  int last;
  float mw[8][kMaxMergeSplits];     // cross-split merge: weight 2^(m_s - M) per head and member
  float Lsum[8];
  float Mmax[8];
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Gather bit p of 8 codes from W plane words (word p at words[p * stride]; code m at bit
// shift + 4m) into 4-bit nibbles: nibble m of the result is code m.
template <int W>
__device__ __forceinline__ uint32_t gather_nibbles(const uint32_t* words, int stride, int shift) {
  uint32_t x = 0;
#pragma unroll
  for (int p = 0; p < W; ++p) x |= rotr(words[p * stride], static_cast<uint32_t>(shift - p) & 31u) & (0x11111111u << p);
  return x;
}

// Register lookup of 8 codes (nibbles of x, each < 8) in an 8-entry fp16 table split into
// low and high bytes; r[k] = fp16x2(entry[code 2k], entry[code 2k+1]).
__device__ __forceinline__ void lut8(uint32_t x, const uint4& L, uint32_t (&r)[4]) {
  const uint32_t la = prmt(L.x, L.y, x), ha = prmt(L.z, L.w, x);
  const uint32_t xh = x >> 16;
  const uint32_t lb = prmt(L.x, L.y, xh), hb = prmt(L.z, L.w, xh);
  r[0] = prmt(la, ha, 0x5140u);
  r[1] = prmt(la, ha, 0x7362u);
  r[2] = prmt(lb, hb, 0x5140u);
  r[3] = prmt(lb, hb, 0x7362u);
}

// 16-entry version: the low 3 bits of a nibble index two 8-entry halves, bit 3 picks the
// half through a byte mask made with prmt's sign-replicate mode.
__device__ __forceinline__ void lut16(uint32_t x, const uint4& LO, const uint4& HI, uint32_t (&r)[4]) {
  const uint32_t x7 = x & 0x77777777u;
  const uint32_t xh = x >> 16, x7h = x7 >> 16;
  const uint32_t ma = prmt(x << 4, x, 0xD9C8u), mb = prmt(xh << 4, xh, 0xD9C8u);
  const uint32_t la = (prmt(LO.x, LO.y, x7) & ~ma) | (prmt(LO.z, LO.w, x7) & ma);
  const uint32_t ha = (prmt(HI.x, HI.y, x7) & ~ma) | (prmt(HI.z, HI.w, x7) & ma);
  const uint32_t lb = (prmt(LO.x, LO.y, x7h) & ~mb) | (prmt(LO.z, LO.w, x7h) & mb);
  const uint32_t hb = (prmt(HI.x, HI.y, x7h) & ~mb) | (prmt(HI.z, HI.w, x7h) & mb);
  r[0] = prmt(la, ha, 0x5140u);
  r[1] = prmt(la, ha, 0x7362u);
  r[2] = prmt(lb, hb, 0x5140u);
  r[3] = prmt(lb, hb, 0x7362u);
}

// Widths 5..8: gather the 8 codes as bytes (even codes in `ev`, odd codes in `od`, byte k =
// code 2k / 2k+1), one rotate + mask per plane and parity, then look each byte up in the
// shared fp16 table.
template <int W>
__device__ __forceinline__ void lut_wide(const uint32_t* words, int stride, int shift, const uint16_t* table,
                                         uint32_t (&r)[4]) {
  uint32_t ev = 0u, od = 0u;
#pragma unroll
  for (int p = 0; p < W; ++p) {
    const uint32_t w = words[p * stride];
    ev |= rotr(w, static_cast<uint32_t>(shift - p) & 31u) & (0x01010101u << p);
    od |= rotr(w, static_cast<uint32_t>(shift + 4 - p) & 31u) & (0x01010101u << p);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k)
    r[k] = pack_u16x2(table[(ev >> (8 * k)) & 0xffu], table[(od >> (8 * k)) & 0xffu]);
}

// The 8 codes of width W at bits shift + 4m of W plane words, as 4 fp16x2 fragments
// (r[k] = (code 2k, code 2k+1)).
template <int W>
__device__ __forceinline__ void decode8(const uint32_t* words, int stride, int shift, const DecodeSmem& S,
                                        uint32_t (&r)[4]) {
  if constexpr (W <= 3) {
    lut8(gather_nibbles<W>(words, stride, shift), S.lut8[W], r);
  } else if constexpr (W == 4) {
    lut16(gather_nibbles<4>(words, stride, shift), S.lut16[0], S.lut16[1], r);
  } else {
    lut_wide<W>(words, stride, shift, S.cent + ((1 << W) - 2), r);
  }
}

// One QK k-step: 4 RoPE blocks (one per lane c) x 32 tokens (4 n-tiles). e = {Q' hi pair,
// Q' lo pair, word offset of this lane's plane-0 word (block offset + half H), unused}.
template <int W>
__device__ __forceinline__ void qk_step(const uint32_t* kw, const uint4& e, int sh, const DecodeSmem& S,
                                        float (&acc)[4][4]) {
  uint32_t bf[4];
  decode8<W>(kw + e.z, 2, sh, S, bf);
#pragma unroll
  for (int j = 0; j < 4; ++j) mma_m16n8k8(acc[j], e.x, e.y, bf[j]);
}

// All k-steps of one width class.
template <int W>
__device__ __forceinline__ void qk_class(const uint32_t* kw, int s0, int s1, int g, int c, int sh,
                                         const DecodeSmem& S, float (&acc)[4][4]) {
  for (int s = s0; s < s1; ++s) qk_step<W>(kw, S.kstep[s][g][c], sh, S, acc);
}

// O += P' V over the 16 dim n-tiles for value width W.
template <int W>
__device__ __forceinline__ void pv_all(const uint32_t* vw, int g, int c, const uint32_t (&pa_hi)[4],
                                       const uint32_t (&pa_lo)[4], const DecodeSmem& S, float (&o_acc)[16][4]) {
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    uint32_t vf[4];
    decode8<W>(vw + 8 * nt + g, kD, c, S, vf);
    mma_m16n8k16(o_acc[nt], pa_hi[0], pa_lo[0], pa_hi[1], pa_lo[1], vf[0], vf[1]);
    mma_m16n8k16(o_acc[nt], pa_hi[2], pa_lo[2], pa_hi[3], pa_lo[3], vf[2], vf[3]);
  }
}

__device__ __forceinline__ void decode_load_tile(uint8_t* dst, const uint8_t* src, int rec_bytes, int lane) {
  for (int k = lane; k < rec_bytes / 16; k += 32) cp_async16(dst + 16 * k, src + 16 * k);
}

// Merge n (m, l, O) partials, entries first..first+n-1 of row `bh` (row pitch `pitch` entries,
// 8 head rows per entry), in entry order: M = max m, L = sum l 2^(m - M),
// O = sum O 2^(m - M). Writes either the merged partial to entry `dst` or, when `out` is
// non-null, out = O / L for the G real heads. Needs all threads of the CTA (256 or 512).
__device__ __forceinline__ void merge_partials(DecodeSmem& S, uint8_t* scratch, int bh, int pitch, int first, int n,
                                               float* part_m, float* part_l, float* part_o, int dst, float* out,
                                               int G) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int hg = warp; hg < 8; hg += kDecWarps) {
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
  // O: 256 (head, 4-dim) quads; with 512 threads two threads share a quad (halves of the
  // member list), with 256 threads one thread does all members.
  const int halves = blockDim.x >> 8;
  const int quad = tid & 255, half = tid >> 8;
  const int hg = quad >> 5, j4 = quad & 31;
  const int s_mid = (halves == 2) ? n / 2 : n;
  const int s0 = half ? s_mid : 0, s1 = half ? n : s_mid;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  const float4* po = reinterpret_cast<const float4*>(part_o);
#pragma unroll 4
  for (int s = s0; s < s1; ++s) {
    const float wt = S.mw[hg][s];
    const float4 v = __ldcg(po + ((static_cast<size_t>(bh) * pitch + first + s) * 8 + hg) * (kD / 4) + j4);
    o.x += v.x * wt; o.y += v.y * wt; o.z += v.z * wt; o.w += v.w * wt;
  }
  float4* red = reinterpret_cast<float4*>(scratch);
  if (half) red[quad] = o;
  __syncthreads();
  if (!half) {
    if (halves == 2) {
      const float4 v = red[quad];
      o.x += v.x; o.y += v.y; o.z += v.z; o.w += v.w;
    }
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
}

template <int DT>
__global__ void __launch_bounds__(kDecWarps * 32) kvq_decode_gtq(
    const typename Elem<DT>::T* __restrict__ q, int64_t qsb, int64_t qsh, int n_q_heads, int n_kv_heads,
    const uint8_t* __restrict__ packed, const kvq_head_alloc* __restrict__ alloc, int tiles_cap,
    int rec_bytes, int bits_v, int seq_len, int splits, int n_groups, int n_stages, float* __restrict__ out,
    float* __restrict__ part_m, float* __restrict__ part_l, float* __restrict__ part_o,
    unsigned* __restrict__ tickets) {
  extern __shared__ __align__(16) uint8_t dsmem[];
  DecodeSmem& S = *reinterpret_cast<DecodeSmem*>(dsmem);
  uint8_t* stages = dsmem + ((sizeof(DecodeSmem) + 127) / 128) * 128;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / n_kv_heads, hkv = bh % n_kv_heads;
  const int G = n_q_heads / n_kv_heads;
  const kvq_head_alloc* al = alloc + hkv;
  const int k_words = al->k_words;
  // An allocation made for another budget does not match the record size: write nothing.
  if (4 * (k_words + bits_v * kD) + 4 * kTile != rec_bytes) return;
  const int n_tiles = (seq_len + kTile - 1) / kTile;
  const int t_begin = static_cast<int>((static_cast<long long>(split) * n_tiles) / splits);
  const int t_end = static_cast<int>((static_cast<long long>(split + 1) * n_tiles) / splits);
  const float inv_sqrt_d = 0.08838834764831845f;

  const int stage_bytes = ((rec_bytes + 127) / 128) * 128;
  uint8_t* my_stages = stages + warp * n_stages * stage_bytes;
  const uint8_t* src_base = packed + static_cast<size_t>(bh) * tiles_cap * rec_bytes;
  const int first = t_begin + warp;
  const int my_n = (first < t_end) ? (t_end - first + kDecWarps - 1) / kDecWarps : 0;
  // Start streaming the first tiles before the prologue.
  for (int i = 0; i < n_stages - 1; ++i) {
    if (i < my_n)
      decode_load_tile(my_stages + i * stage_bytes, src_base + static_cast<size_t>(first + i * kDecWarps) * rec_bytes,
                       rec_bytes, lane);
    cp_async_commit();
  }

  // ------------------------------------------------------------------ prologue
  for (int i = tid; i < kCentroidCount; i += blockDim.x) S.cent[i] = c_tab.centroid_f16[i];
  if (tid < 4) {
    uint32_t lo[2] = {0u, 0u}, hi[2] = {0u, 0u};
    if (tid >= 1) {
      for (int e = 0; e < (1 << tid); ++e) {
        const uint32_t c16 = c_tab.centroid_f16[(1 << tid) - 2 + e];
        lo[e >> 2] |= (c16 & 0xffu) << (8 * (e & 3));
        hi[e >> 2] |= (c16 >> 8) << (8 * (e & 3));
      }
    }
    S.lut8[tid] = make_uint4(lo[0], lo[1], hi[0], hi[1]);
  } else if (tid == 4) {
    uint32_t lo[4] = {0u, 0u, 0u, 0u}, hi[4] = {0u, 0u, 0u, 0u};
    for (int e = 0; e < 16; ++e) {
      const uint32_t c16 = c_tab.centroid_f16[14 + e];
      lo[e >> 2] |= (c16 & 0xffu) << (8 * (e & 3));
      hi[e >> 2] |= (c16 >> 8) << (8 * (e & 3));
    }
    S.lut16[0] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    S.lut16[1] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
  }
  for (int i = tid; i < kH; i += blockDim.x) S.woff[i] = al->word_off[i];
  for (int i = tid; i < kMaxSteps * 4; i += blockDim.x) S.step_blk[i >> 2][i & 3] = al->step_block[i >> 2][i & 3];
  for (int i = tid; i < kMaxSteps; i += blockDim.x) S.step_w[i] = al->step_width[i];
  if (tid == 0) S.n_steps = min(max(al->n_steps, 0), kMaxSteps);
  for (int i = tid; i < 8 * kD; i += blockDim.x) {
    const int hg = i / kD, j = i % kD;
    float v = 0.0f;
    if (hg < G) {
      const float qv = Elem<DT>::to_f32(q[b * qsb + (hkv * G + hg) * qsh + j]);
      v = qv * al->dequant[j % kH] * (inv_sqrt_d * kLog2e);
    }
    S.qp[hg][j] = v;
  }
  __syncthreads();
  // per-head power-of-two scaling so the largest |Q'| lies in [0.5, 1)
  for (int hg = warp; hg < 8; hg += kDecWarps) {
    float mx = 0.0f;
    for (int j = lane; j < kD; j += 32) mx = fmaxf(mx, fabsf(S.qp[hg][j]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    int e = 0;
    if (mx > 0.0f) frexpf(mx, &e);
    if (lane == 0) S.qmul[hg] = ldexpf(1.0f, e);
    const float sc = ldexpf(1.0f, -e);
    for (int j = lane; j < kD; j += 32) S.qp[hg][j] *= sc;
  }
  __syncthreads();
  const int n_steps = S.n_steps;
  for (int i = tid; i < n_steps * 32; i += blockDim.x) {
    const int st = i >> 5, hg = (i >> 2) & 7, cc = i & 3;
    const int blk = S.step_blk[st][cc];
    uint4 e = make_uint4(0u, 0u, 0u, 0u);
    int wblk = blk;
    if (blk >= 0 && blk < kH) {
      __half h1, l1, h2, l2;
      split_hilo(S.qp[hg][blk], h1, l1);
      split_hilo(S.qp[hg][blk + kH], h2, l2);
      e.x = pack_half2(h1, h2);
      e.y = pack_half2(l1, l2);
    } else {
      wblk = max(static_cast<int>(S.step_blk[st][0]), 0);   // empty slot: Q' is 0, read any valid block
    }
    e.z = static_cast<uint32_t>(S.woff[min(wblk, kH - 1)]) + (hg >> 2);   // lane (hg, cc) uses half H = hg / 4
    S.kstep[st][hg][cc] = e;
  }
  if (tid == 0) {
    int n = 0;
    for (int st = 0; st < n_steps; ++st) {
      const int w = min(max(static_cast<int>(S.step_w[st]), 1), 8);
      if (n == 0 || S.cls_w[n - 1] != w) {
        S.cls_w[n] = w;
        S.cls_begin[n] = st;
        ++n;
      }
    }
    S.cls_begin[n] = n_steps;
    S.n_cls = n;
  }
  __syncthreads();

  // ------------------------------------------------------------------ main loop
  const float qmul = S.qmul[g];
  float m_run = -INFINITY, l_run = 0.0f;
  float o_acc[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) o_acc[nt][0] = o_acc[nt][1] = o_acc[nt][2] = o_acc[nt][3] = 0.0f;

  const int sh = g & 3;
  for (int i = 0; i < my_n; ++i) {
    {
      const int nxt = i + n_stages - 1;
      if (nxt < my_n)
        decode_load_tile(my_stages + (nxt % n_stages) * stage_bytes,
                         src_base + static_cast<size_t>(first + nxt * kDecWarps) * rec_bytes, rec_bytes, lane);
      cp_async_commit();
    }
    cp_async_wait_pending(n_stages - 1);
    __syncwarp();
    const int tile = first + i * kDecWarps;
    const uint8_t* st = my_stages + (i % n_stages) * stage_bytes;
    const uint32_t* kw = reinterpret_cast<const uint32_t*>(st);
    const uint32_t* vw = kw + k_words;
    const uint16_t* kn = reinterpret_cast<const uint16_t*>(vw + bits_v * kD);
    const uint16_t* vn = kn + kTile;

    // ---- S^T = Q' K^T over the k-steps
    float acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
    for (int ci = 0; ci < S.n_cls; ++ci) {
      const int s0 = S.cls_begin[ci], s1 = S.cls_begin[ci + 1];
      switch (S.cls_w[ci]) {
        case 1: qk_class<1>(kw, s0, s1, g, c, sh, S, acc); break;
        case 2: qk_class<2>(kw, s0, s1, g, c, sh, S, acc); break;
        case 3: qk_class<3>(kw, s0, s1, g, c, sh, S, acc); break;
        case 4: qk_class<4>(kw, s0, s1, g, c, sh, S, acc); break;
        case 5: qk_class<5>(kw, s0, s1, g, c, sh, S, acc); break;
        case 6: qk_class<6>(kw, s0, s1, g, c, sh, S, acc); break;
        case 7: qk_class<7>(kw, s0, s1, g, c, sh, S, acc); break;
        default: qk_class<8>(kw, s0, s1, g, c, sh, S, acc); break;
      }
    }

    // ---- online softmax over the 8 tokens this lane holds: 8j + 2c + {0,1}
    float sv[4][2];
    float tmax = -INFINITY;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int tt = 8 * j + 2 * c + u;
        const float nk = __half2float(__ushort_as_half(kn[tt]));
        float sval = (acc[j][u] + acc[j][u + 2]) * nk * qmul;
        if (tile * kTile + tt >= seq_len) sval = -INFINITY;
        sv[j][u] = sval;
        tmax = fmaxf(tmax, sval);
      }
    }
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
    const float m_new = fmaxf(m_run, tmax);
    const float alpha = (m_run == -INFINITY) ? 0.0f : fast_exp2(m_run - m_new);
    m_run = m_new;
    l_run *= alpha;
    if (!__all_sync(0xffffffffu, alpha == 1.0f)) {
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        o_acc[nt][0] *= alpha; o_acc[nt][1] *= alpha; o_acc[nt][2] *= alpha; o_acc[nt][3] *= alpha;
      }
    }
    uint32_t pa_hi[4], pa_lo[4];   // per n-tile j: packed (token 8j+2c, 8j+2c+1)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      __half hh[2], ll[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int tt = 8 * j + 2 * c + u;
        const float p = (sv[j][u] == -INFINITY) ? 0.0f : fast_exp2(sv[j][u] - m_new);
        l_run += p;
        const float pv = p * __half2float(__ushort_as_half(vn[tt])) * inv_sqrt_d;
        split_hilo(pv, hh[u], ll[u]);
      }
      pa_hi[j] = pack_half2(hh[0], hh[1]);
      pa_lo[j] = pack_half2(ll[0], ll[1]);
    }

    // ---- O += P' Vhat over 16 dim n-tiles, two 16-token k-steps
    switch (bits_v) {
      case 1: pv_all<1>(vw, g, c, pa_hi, pa_lo, S, o_acc); break;
      case 2: pv_all<2>(vw, g, c, pa_hi, pa_lo, S, o_acc); break;
      case 3: pv_all<3>(vw, g, c, pa_hi, pa_lo, S, o_acc); break;
      case 4: pv_all<4>(vw, g, c, pa_hi, pa_lo, S, o_acc); break;
      case 5: pv_all<5>(vw, g, c, pa_hi, pa_lo, S, o_acc); break;
      case 6: pv_all<6>(vw, g, c, pa_hi, pa_lo, S, o_acc); break;
      case 7: pv_all<7>(vw, g, c, pa_hi, pa_lo, S, o_acc); break;
      default: pv_all<8>(vw, g, c, pa_hi, pa_lo, S, o_acc); break;
    }
    __syncwarp();
  }
  cp_async_wait_pending(0);

  // ------------------------------------------------------------------ combine warps
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  __syncthreads();
  float* cm = reinterpret_cast<float*>(stages);                  // [4][8]
  float* cl = cm + kDecWarps * 8;                                 // [4][8]
  float* co = cl + kDecWarps * 8;                                 // [4][8][128]
  if (c == 0) {
    cm[warp * 8 + g] = m_run;
    cl[warp * 8 + g] = l_run;
  }
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    co[(warp * 8 + g) * kD + 8 * nt + 2 * c] = o_acc[nt][0] + o_acc[nt][2];
    co[(warp * 8 + g) * kD + 8 * nt + 2 * c + 1] = o_acc[nt][1] + o_acc[nt][3];
  }
  __syncthreads();
  for (int i = tid; i < 8 * kD; i += blockDim.x) {
    const int hg = i / kD, j = i % kD;
    float M = -INFINITY;
    for (int wv = 0; wv < kDecWarps; ++wv) M = fmaxf(M, cm[wv * 8 + hg]);
    float L = 0.0f, O = 0.0f;
    for (int wv = 0; wv < kDecWarps; ++wv) {
      const float mw = cm[wv * 8 + hg];
      const float wt = (mw == -INFINITY) ? 0.0f : fast_exp2(mw - M);
      L += cl[wv * 8 + hg] * wt;
      O += co[(wv * 8 + hg) * kD + j] * wt;
    }
    if (splits == 1) {
      if (hg < G) out[(static_cast<size_t>(b) * n_q_heads + hkv * G + hg) * kD + j] = O / L;
    } else {
      const size_t pb = (static_cast<size_t>(bh) * (splits + n_groups) + split) * 8 + hg;
      part_o[pb * kD + j] = O;
      if (j == 0) {
        part_m[pb] = M;
        part_l[pb] = L;
      }
    }
  }
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
