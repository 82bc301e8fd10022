// Calibration kernels: the label-free energy score per RoPE block and the greedy integer
// bit allocation by marginal gain ("RoPE-aware bit allocation for KV cache quantization",
// abstract: "for each layer and KV head, Block-GTQ computes a label-free energy score for
// each RoPE block and greedily allocates integer bit widths by marginal gain").
#pragma once

#include "common.cuh"

namespace kvq {

// One warp per (64-token chunk, KV head). Lane l owns blocks 2l and 2l+1, i.e. dims
// (2l, 2l+1) and (64+2l, 65+2l), read as one 2-element vector each (coalesced 128 B per
// warp-load for 16-bit inputs). Within the chunk the pooled tokens u = s*n_calib + t are
// summed left to right in fp64, each term being fl(fl(x^2) + fl(y^2)).
template <int DT>
__global__ void __launch_bounds__(32) kvq_calib_reduce(const typename Elem<DT>::T* __restrict__ K,
                                                       int n_calib, int64_t sb, int64_t sh, int64_t st,
                                                       int N, int n_chunks, double* __restrict__ partial) {
  using T = typename Elem<DT>::T;
  const int c = blockIdx.x, h = blockIdx.y, l = threadIdx.x;
  const int u0 = c * kCalibChunk;
  const int u1 = min(N, u0 + kCalibChunk);
  double acc0 = 0.0, acc1 = 0.0;
#pragma unroll 8
  for (int u = u0; u < u1; ++u) {
    const int s = u / n_calib;
    const int t = u - s * n_calib;
    const T* row = K + s * sb + h * sh + static_cast<int64_t>(t) * st;
    float x0, x1, y0, y1;
    if constexpr (DT == KVQ_F32) {
      const float2 a = *reinterpret_cast<const float2*>(row + 2 * l);
      const float2 b = *reinterpret_cast<const float2*>(row + kH + 2 * l);
      x0 = a.x; x1 = a.y; y0 = b.x; y1 = b.y;
    } else {
      const T* pa = row + 2 * l;
      const T* pb = row + kH + 2 * l;
      x0 = Elem<DT>::to_f32(pa[0]); x1 = Elem<DT>::to_f32(pa[1]);
      y0 = Elem<DT>::to_f32(pb[0]); y1 = Elem<DT>::to_f32(pb[1]);
    }
    const double dx0 = x0, dx1 = x1, dy0 = y0, dy1 = y1;
    acc0 = __dadd_rn(acc0, __dadd_rn(__dmul_rn(dx0, dx0), __dmul_rn(dy0, dy0)));
    acc1 = __dadd_rn(acc1, __dadd_rn(__dmul_rn(dx1, dx1), __dmul_rn(dy1, dy1)));
  }
  double* dst = partial + (static_cast<size_t>(h) * n_chunks + c) * kH;
  dst[2 * l] = acc0;
  dst[2 * l + 1] = acc1;
}

// One CTA of 512 threads per KV head.
//  1. E_b = (sum of chunk partials, left to right) / N, fp64.
//  2. Greedy allocation in rank form: entry e = 8b + w (w < w_max) has marginal gain
//     E_b (delta(w) - delta(w+1)); the greedy takes the bits_k * 64 first entries in the
//     order (gain descending, e ascending). Because delta is strictly convex each block's
//     gains are non-increasing in w, so this is the step-by-step greedy with ties to the
//     lowest block, and the picked entries of a block are a prefix: w_b = their count.
//  3. g_b, f_b, the K word offsets and the decode k-step table (blocks grouped by width,
//     widest first, 4 per step, ascending block index within a width).
__global__ void __launch_bounds__(512) kvq_greedy_alloc(const double* __restrict__ partial, int n_chunks,
                                                        int N, int bits_k, int w_max, int mode,
                                                        kvq_head_alloc* __restrict__ alloc) {
  __shared__ double sE[kH];
  __shared__ double sGain[kH * 8];
  __shared__ int sWidth[kH];
  __shared__ float sG[kH];
  __shared__ int sStepStart[9];
  __shared__ int sCount[9];
  __shared__ double sSum;
  const int h = blockIdx.x, tid = threadIdx.x;
  kvq_head_alloc* al = alloc + h;

  if (tid < kH) {
    double S = 0.0;
    const double* p = partial + static_cast<size_t>(h) * n_chunks * kH + tid;
    for (int c = 0; c < n_chunks; ++c) S = __dadd_rn(S, p[static_cast<size_t>(c) * kH]);
    sE[tid] = __ddiv_rn(S, static_cast<double>(N));
  }
  __syncthreads();
  if (tid == 0) {
    double S = 0.0;
    for (int b = 0; b < kH; ++b) S = __dadd_rn(S, sE[b]);
    sSum = S;
  }
  {
    const int b = tid >> 3, w = tid & 7;
    const bool valid = w < w_max;
    sGain[tid] = valid ? __dmul_rn(sE[b], __dsub_rn(static_cast<double>(c_tab.delta[w]),
                                                    static_cast<double>(c_tab.delta[w + 1])))
                       : -1.0;
  }
  __syncthreads();
  if (mode == KVQ_MODE_UNIFORM) {
    if (tid < kH) sWidth[tid] = bits_k;
  } else {
    const double gain = sGain[tid];
    const bool valid = (tid & 7) < w_max;
    int rank = 0;
    for (int e = 0; e < kH * 8; ++e) {
      const double ge = sGain[e];
      rank += (ge > gain) || (ge == gain && e < tid);
    }
    const bool picked = valid && rank < bits_k * kH;
    const unsigned mask = __ballot_sync(0xffffffffu, picked);
    if ((tid & 7) == 0) sWidth[tid >> 3] = __popc((mask >> (tid & 24)) & 0xffu);
  }
  if (tid < 9) sCount[tid] = 0;
  __syncthreads();

  if (tid < kH) {
    const int b = tid;
    float g = 1.0f;
    if (mode != KVQ_MODE_UNIFORM && sE[b] > 0.0 && sSum > 0.0)
      g = __double2float_rn(__dsqrt_rn(__ddiv_rn(__dmul_rn(2.0, sSum), __dmul_rn(static_cast<double>(kD), sE[b]))));
    sG[b] = g;
    al->energy[b] = sE[b];
    al->gain[b] = g;
    al->dequant[b] = __double2float_rn(__ddiv_rn(1.0, __dmul_rn(__dsqrt_rn(static_cast<double>(kD)),
                                                                static_cast<double>(g))));
    al->width[b] = static_cast<uint8_t>(sWidth[b]);
    atomicAdd(&sCount[sWidth[b]], 1);
  }
  if (tid < 32 * 4) {
    al->step_block[tid >> 2][tid & 3] = -1;
  }
  if (tid >= 128 && tid < 160) al->step_width[tid - 128] = 0;
  __syncthreads();
  if (tid == 0) {
    int off = 0;
    for (int b = 0; b < kH; ++b) {
      al->word_off[b] = static_cast<uint16_t>(off);
      off += 2 * sWidth[b];
    }
    int steps = 0;
    for (int w = 8; w >= 1; --w) {
      sStepStart[w] = steps;
      steps += (sCount[w] + 3) / 4;
    }
    sStepStart[0] = steps;
    al->n_steps = steps;
    al->k_words = off;
    al->head_dim = kD;
    al->bits_k = bits_k;
    al->w_max = w_max;
    al->mode = mode;
    al->reserved[0] = 0;
    al->reserved[1] = 0;
  }
  __syncthreads();
  if (tid < kH) {
    const int b = tid, w = sWidth[b];
    if (w > 0) {
      int r = 0;
      for (int j = 0; j < b; ++j) r += (sWidth[j] == w);
      const int s = sStepStart[w] + r / 4;
      al->step_block[s][r & 3] = static_cast<int8_t>(b);
      al->step_width[s] = static_cast<uint8_t>(w);
    }
  }
}

}  // namespace kvq
