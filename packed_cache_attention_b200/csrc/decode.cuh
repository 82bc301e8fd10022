// Fused decode attention read straight from the packed Block-GTQ cache ("RoPE-aware bit
// allocation for KV cache quantization", abstract: "packed-cache serving path"; the NQKV
// review's editorial extension: fuse the table lookup into the attention kernel).
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

constexpr int kDecWarps = 4;
constexpr int kDecStages = 3;
constexpr int kMaxSteps = 32;
constexpr int kTargetCtas = 296;   // 2 CTAs per SM on a 148-SM B200

struct DecodeSmem {
  uint2 qfrag[kMaxSteps][8][4];     // A fragments of Q' per k-step, head row g, lane c
  float qp[8][kD];                  // Q' in fp32 before scaling
  float qmul[8];                    // 2^e that undoes the per-head scaling of Q'
  uint16_t cent[kCentroidCount];    // fp16 centroid bit patterns
  uint16_t woff[kH];
  int8_t step_blk[kMaxSteps][4];
  uint8_t step_w[kMaxSteps];
  int n_steps;
  int last;
};

__device__ __forceinline__ void decode_load_tile(uint8_t* dst, const uint8_t* src, int rec_bytes, int lane) {
  for (int k = lane; k < rec_bytes / 16; k += 32) cp_async16(dst + 16 * k, src + 16 * k);
}

template <int DT>
__global__ void __launch_bounds__(kDecWarps * 32) kvq_decode_gtq(
    const typename Elem<DT>::T* __restrict__ q, int64_t qsb, int64_t qsh, int n_q_heads, int n_kv_heads,
    const uint8_t* __restrict__ packed, const kvq_head_alloc* __restrict__ alloc, int tiles_cap,
    int rec_bytes, int bits_v, int seq_len, int splits, float* __restrict__ out,
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

  // ------------------------------------------------------------------ prologue
  for (int i = tid; i < kCentroidCount; i += blockDim.x) S.cent[i] = c_tab.centroid_f16[i];
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
    const int s = i >> 5, hg = (i >> 2) & 7, cc = i & 3;
    const int blk = S.step_blk[s][cc];
    uint2 fr = make_uint2(0u, 0u);
    if (blk >= 0 && blk < kH) {
      __half h1, l1, h2, l2;
      split_hilo(S.qp[hg][blk], h1, l1);
      split_hilo(S.qp[hg][blk + kH], h2, l2);
      fr.x = pack_half2(h1, h2);
      fr.y = pack_half2(l1, l2);
    }
    S.qfrag[s][hg][cc] = fr;
  }
  __syncthreads();

  // ------------------------------------------------------------------ main loop
  const float qmul = S.qmul[g];
  float m_run = -INFINITY, l_run = 0.0f;
  float o_acc[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) o_acc[nt][0] = o_acc[nt][1] = o_acc[nt][2] = o_acc[nt][3] = 0.0f;

  const int stage_bytes = ((rec_bytes + 127) / 128) * 128;
  uint8_t* my_stages = stages + warp * kDecStages * stage_bytes;
  const uint8_t* src_base = packed + static_cast<size_t>(bh) * tiles_cap * rec_bytes;
  const int first = t_begin + warp;
  const int my_n = (first < t_end) ? (t_end - first + kDecWarps - 1) / kDecWarps : 0;

#pragma unroll
  for (int i = 0; i < kDecStages - 1; ++i) {
    if (i < my_n)
      decode_load_tile(my_stages + i * stage_bytes, src_base + static_cast<size_t>(first + i * kDecWarps) * rec_bytes,
                       rec_bytes, lane);
    cp_async_commit();
  }

  const int H = g >> 2, sh = g & 3;
  for (int i = 0; i < my_n; ++i) {
    {
      const int nxt = i + kDecStages - 1;
      if (nxt < my_n)
        decode_load_tile(my_stages + (nxt % kDecStages) * stage_bytes,
                         src_base + static_cast<size_t>(first + nxt * kDecWarps) * rec_bytes, rec_bytes, lane);
      cp_async_commit();
    }
    cp_async_wait<kDecStages - 1>();
    __syncwarp();
    const int tile = first + i * kDecWarps;
    const uint8_t* st = my_stages + (i % kDecStages) * stage_bytes;
    const uint32_t* kw = reinterpret_cast<const uint32_t*>(st);
    const uint32_t* vw = kw + k_words;
    const uint16_t* kn = reinterpret_cast<const uint16_t*>(vw + bits_v * kD);
    const uint16_t* vn = kn + kTile;

    // ---- S^T = Q' K^T over the k-steps
    float acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
    for (int s = 0; s < n_steps; ++s) {
      const int w = min(max(static_cast<int>(S.step_w[s]), 1), 8);
      int blk = S.step_blk[s][c];
      if (blk < 0) blk = max(static_cast<int>(S.step_blk[s][0]), 0);   // empty slot: Q' is 0 there
      const uint32_t* bw = kw + S.woff[blk] + H;
      uint32_t W[8];
#pragma unroll
      for (int p = 0; p < 8; ++p) W[p] = (p < w) ? bw[2 * p] : 0u;
      const uint16_t* cb = S.cent + ((1 << w) - 2);
      uint32_t val[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        int code = 0;
#pragma unroll
        for (int p = 0; p < 8; ++p) code |= ((W[p] >> (sh + 4 * m)) & 1u) << p;
        val[m] = cb[code];
      }
      const uint2 a = S.qfrag[s][g][c];
#pragma unroll
      for (int j = 0; j < 4; ++j) mma_m16n8k8(acc[j], a.x, a.y, pack_u16x2(val[2 * j], val[2 * j + 1]));
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
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      o_acc[nt][0] *= alpha; o_acc[nt][1] *= alpha; o_acc[nt][2] *= alpha; o_acc[nt][3] *= alpha;
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
    const uint16_t* vcb = S.cent + ((1 << bits_v) - 2);
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int jd = 8 * nt + g;
      uint32_t W[8];
#pragma unroll
      for (int p = 0; p < 8; ++p) W[p] = (p < bits_v) ? vw[p * kD + jd] : 0u;
      uint32_t val[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        int code = 0;
#pragma unroll
        for (int p = 0; p < 8; ++p) code |= ((W[p] >> (c + 4 * m)) & 1u) << p;
        val[m] = vcb[code];
      }
      mma_m16n8k16(o_acc[nt], pa_hi[0], pa_lo[0], pa_hi[1], pa_lo[1], pack_u16x2(val[0], val[1]),
                   pack_u16x2(val[2], val[3]));
      mma_m16n8k16(o_acc[nt], pa_hi[2], pa_lo[2], pa_hi[3], pa_lo[3], pack_u16x2(val[4], val[5]),
                   pack_u16x2(val[6], val[7]));
    }
    __syncwarp();
  }
  cp_async_wait<0>();

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
      const size_t pb = (static_cast<size_t>(bh) * splits + split) * 8 + hg;
      part_o[pb * kD + j] = O;
      if (j == 0) {
        part_m[pb] = M;
        part_l[pb] = L;
      }
    }
  }
  if (splits == 1) return;

  // ------------------------------------------------------------------ cross-split merge
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned ticket = atomicAdd(&tickets[bh], 1u);
    S.last = (ticket == static_cast<unsigned>(splits - 1));
  }
  __syncthreads();
  if (!S.last) return;
  __threadfence();
  for (int i = tid; i < 8 * kD; i += blockDim.x) {
    const int hg = i / kD, j = i % kD;
    if (hg >= G) continue;
    const size_t p0 = static_cast<size_t>(bh) * splits * 8 + hg;
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, __ldcg(part_m + p0 + static_cast<size_t>(s) * 8));
    float L = 0.0f, O = 0.0f;
    for (int s = 0; s < splits; ++s) {
      const size_t pi = p0 + static_cast<size_t>(s) * 8;
      const float ms = __ldcg(part_m + pi);
      const float wt = (ms == -INFINITY) ? 0.0f : fast_exp2(ms - M);
      L += __ldcg(part_l + pi) * wt;
      O += __ldcg(part_o + pi * kD + j) * wt;
    }
    out[(static_cast<size_t>(b) * n_q_heads + hkv * G + hg) * kD + j] = O / L;
  }
  if (tid == 0) tickets[bh] = 0u;
}

}  // namespace kvq
