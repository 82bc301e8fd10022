// NQKV-style NF4 variant (review of "NQKV: A KV Cache Quantization Scheme Based on Normal
// Distribution Characteristics": 256-value blocks along each token's hidden vector, a
// block scale from the maximum absolute value with no mean subtraction, 4-bit NF4
// indices, dequantization by table lookup, token rows padded to a multiple of 16).
//
// Buffer layout (nblk = n_heads * 128 / 256 blocks per token, T_pad = ceil(capacity/16)*16):
//   K codes [batch][nblk][T_pad][128 B] | V codes (same) | K scales [batch][nblk][T_pad] fp16
//   | V scales (same). Byte k of a row holds value 2k (low nibble) and 2k+1 (high nibble);
//   block blk of a token covers heads 2*blk (values 0..127) and 2*blk+1 (values 128..255).
#pragma once

#include <cmath>
#include <cstring>

#include "common.cuh"

namespace kvq {

constexpr int kNf4Warps = 8;

struct Nf4Layout {
  int nblk, t_pad;
  size_t codes_bytes;   // one of K/V
  __host__ __device__ size_t row(int b, int blk, int t) const {
    return (static_cast<size_t>(b) * nblk + blk) * t_pad + t;
  }
};

// Index search: u = x / scale lies in [-1, 1] (up to the fp16 rounding of the scale). A
// table cuts [-1, 1) into 32 cells of 1/16, narrower than the smallest gap between the stored
// midpoints, so a cell holds at most one; entry {below, tau} of a cell is the number of
// midpoints below its left edge and the midpoint inside it (+inf if none), and the index
// #{midpoints < u} is below + (u > tau). The cell comes from v = u/2 + 1/2 rounded down and
// saturated to [0, 1] (NaN to 0), then floor(32 v) from a second round-down multiply-add
// against 1.5 * 2^23: both steps round down at power-of-two scales, so the cell is exactly
// the real u's cell; u >= 1 lands in the extra cell 32 (all midpoints below).
constexpr int kNf4LutCells = 33;

// Host: the index table from the 15 fp32 midpoints; false if a cell would hold two or a
// midpoint lies outside [-1, 1).
inline bool nf4_lut_image(const float* mid, uint32_t* out /* 2 * kNf4LutCells */) {
  if (static_cast<double>(mid[0]) < -1.0 || static_cast<double>(mid[14]) >= 1.0) return false;
  for (int k = 0; k < kNf4LutCells; ++k) {
    const double lo = -1.0 + k / 16.0, hi = (k == kNf4LutCells - 1) ? INFINITY : lo + 1.0 / 16.0;
    uint32_t below = 0, inside = 0, tau = 0x7f800000u;
    for (int i = 0; i < 15; ++i) {
      const double m = mid[i];
      if (m < lo) ++below;
      else if (m < hi) {
        ++inside;
        std::memcpy(&tau, &mid[i], 4);
      }
    }
    if (inside > 1) return false;
    out[2 * k] = below;
    out[2 * k + 1] = tau;
  }
  return true;
}

__device__ __align__(16) uint32_t g_nf4_lut[2 * kNf4LutCells];

// NF4 index of u from the table in shared memory (lut_s: its shared-memory address).
__device__ __forceinline__ uint32_t nf4_index(float u, uint32_t lut_s) {
  float v;
  asm("fma.rm.sat.f32 %0, %1, 0f3F000000, 0f3F000000;" : "=f"(v) : "f"(u));
  const float f = __fmaf_rd(v, 32.0f, 12582912.0f);
  const uint32_t addr = static_cast<uint32_t>(__float_as_int(f)) * 8u + (lut_s - 8u * 0x4B400000u);
  uint32_t below, tau;
  asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(below), "=r"(tau) : "r"(addr));
  return below + (u > __uint_as_float(tau) ? 1u : 0u);
}

constexpr int kNf4Rows = 4;   // token rows per warp task
constexpr int kNf4DecWarps = 8;    // warps per CTA of the NF4 decode (four CTAs per SM)
constexpr int kNf4MaxSplits = 160;  // splits per (sequence, head) the NF4 merge reads

// One warp per (K-or-V, sequence, block, group of 4 token rows). Lane l holds values 8l..8l+7
// of the block: head 2*blk + l/16, dims 8(l%16)..8(l%16)+7. All rows of the group are loaded
// before any is quantized. Rows t_begin .. t_end - 1 are quantized (input row i holds token
// t_begin + i), rows t_end .. t_stop - 1 are written as padding (code 0, scale 0), and rows
// outside [t_begin, t_stop) are not touched. kRange = false (a whole-cache quantize: t_begin
// = 0, t_stop = T_pad) compiles without the range checks.
template <int DT, bool kRange>
__global__ void __launch_bounds__(kNf4Warps * 32, 4) kvq_nf4_quant_pack(
    const typename Elem<DT>::T* __restrict__ K, int64_t ksb, int64_t ksh, int64_t kst,
    const typename Elem<DT>::T* __restrict__ V, int64_t vsb, int64_t vsh, int64_t vst, int batch,
    int t_begin, int t_end, int t_stop, Nf4Layout L, uint8_t* __restrict__ packed) {
  using T = typename Elem<DT>::T;
  __shared__ uint2 sLut[kNf4LutCells];
  if (threadIdx.x < kNf4LutCells) sLut[threadIdx.x] = make_uint2(g_nf4_lut[2 * threadIdx.x], g_nf4_lut[2 * threadIdx.x + 1]);
  __syncthreads();
  const uint32_t lut_s = static_cast<uint32_t>(__cvta_generic_to_shared(sLut));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g_lo = t_begin / kNf4Rows;
  const int groups = (t_stop + kNf4Rows - 1) / kNf4Rows - g_lo;
  const long long task = static_cast<long long>(blockIdx.x) * kNf4Warps + warp;
  const long long per_kv = static_cast<long long>(batch) * L.nblk * groups;
  if (task >= 2 * per_kv) return;
  const int which = static_cast<int>(task / per_kv);          // 0 = K, 1 = V
  long long r = task % per_kv;
  const int grp = g_lo + static_cast<int>(r % groups);
  r /= groups;
  const int blk = static_cast<int>(r % L.nblk);
  const int b = static_cast<int>(r / L.nblk);
  const T* X = which ? V : K;
  const int64_t sb = which ? vsb : ksb, sh = which ? vsh : ksh, st = which ? vst : kst;
  const int head = 2 * blk + (lane >> 4), d0 = 8 * (lane & 15);
  const int t0 = grp * kNf4Rows;
  float x[kNf4Rows][8];
#pragma unroll
  for (int rr = 0; rr < kNf4Rows; ++rr) {
    const int t = t0 + rr;
#pragma unroll
    for (int i = 0; i < 8; ++i) x[rr][i] = 0.0f;
    if ((!kRange || t >= t_begin) && t < t_end) {
      const T* src = X + b * sb + head * sh + static_cast<int64_t>(t - t_begin) * st + d0;
      if constexpr (DT == KVQ_F32) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(src));
        const float4 c = __ldg(reinterpret_cast<const float4*>(src) + 1);
        x[rr][0] = a.x; x[rr][1] = a.y; x[rr][2] = a.z; x[rr][3] = a.w;
        x[rr][4] = c.x; x[rr][5] = c.y; x[rr][6] = c.z; x[rr][7] = c.w;
      } else {
        const uint4 a = __ldg(reinterpret_cast<const uint4*>(src));
        const uint32_t wv[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          x[rr][2 * i] = Elem<DT>::to_f32(bits_to<T>(wv[i] & 0xffffu));
          x[rr][2 * i + 1] = Elem<DT>::to_f32(bits_to<T>(wv[i] >> 16));
        }
      }
    }
  }
#pragma unroll
  for (int rr = 0; rr < kNf4Rows; ++rr) {
    const int t = t0 + rr;
    if (kRange && (t < t_begin || t >= t_stop)) continue;   // warp-uniform
    const size_t row = L.row(b, blk, t);
    uint32_t* codes = reinterpret_cast<uint32_t*>(packed + which * L.codes_bytes + row * 128);
    __half* scales = reinterpret_cast<__half*>(packed + 2 * L.codes_bytes) + which * (L.codes_bytes / 128) + row;
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(x[rr][i]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const __half s16 = __float2half_rn(amax);        // padding rows are all zero: scale 0, codes 0
    const float s = __half2float(s16);
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float u = (s == 0.0f) ? 0.0f : __fdiv_rn(x[rr][i], s);
      word |= nf4_index(u, lut_s) << (4 * i);
    }
    if (t >= t_end) word = 0u;
    codes[lane] = word;
    if (lane == 0) *scales = (t < t_end) ? s16 : __ushort_as_half(0);
  }
}

// MHA decode (G = 1), CUDA cores. Grid (splits, batch * n_heads), kNf4DecWarps warps per CTA,
// each warp every kNf4DecWarps-th 32-token group of the CTA's range. Q.K: lane t scores token t of the
// group from its 64 code bytes; P.V: lane l accumulates dims 4l..4l+3 over the group.
template <int DT>
__global__ void __launch_bounds__(kNf4DecWarps * 32) kvq_nf4_decode(
    const typename Elem<DT>::T* __restrict__ q, int64_t qsb, int64_t qsh, int n_heads, const uint8_t* __restrict__ packed,
    Nf4Layout L, int seq_len, int splits, float* __restrict__ out, float* __restrict__ part_m,
    float* __restrict__ part_l, float* __restrict__ part_o, unsigned* __restrict__ tickets) {
  __shared__ float sQ[kD];
  __shared__ float sLut[16];
  __shared__ float cm[kNf4DecWarps], cl[kNf4DecWarps];
  __shared__ float co[kNf4DecWarps][kD];
  __shared__ int sLast;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / n_heads, hh = bh % n_heads;
  const int blk = hh >> 1, half_off = 64 * (hh & 1);
  const float scl = 0.08838834764831845f * kLog2e;
  if (tid < kD) sQ[tid] = Elem<DT>::to_f32(q[b * qsb + hh * qsh + tid]) * scl;
  if (tid < 16) sLut[tid] = c_tab.nf4[tid];
  __syncthreads();

  const int n_groups = (seq_len + 31) / 32;
  const int g0 = static_cast<int>((static_cast<long long>(split) * n_groups) / splits);
  const int g1 = static_cast<int>((static_cast<long long>(split + 1) * n_groups) / splits);
  const uint8_t* kc = packed;
  const uint8_t* vc = packed + L.codes_bytes;
  const __half* ks = reinterpret_cast<const __half*>(packed + 2 * L.codes_bytes);
  const __half* vs = ks + L.codes_bytes / 128;

  float m_run = -INFINITY, l_run = 0.0f, o[4] = {0.f, 0.f, 0.f, 0.f};
  for (int grp = g0 + warp; grp < g1; grp += kNf4DecWarps) {
    const int t = grp * 32 + lane;
    float logit = -INFINITY;
    if (t < seq_len) {
      const size_t row = L.row(b, blk, t);
      const uint4* kr = reinterpret_cast<const uint4*>(kc + row * 128 + half_off);
      // four partial sums (dims 8k'..8k'+7 of each 32-dim quarter go to sum k') keep the
      // dependent chain short; they are added at the end.
      uint4 w4[4];
#pragma unroll
      for (int v = 0; v < 4; ++v) w4[v] = __ldg(kr + v);
      float acc4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint32_t ws[4] = {w4[v].x, w4[v].y, w4[v].z, w4[v].w};
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
          for (int n = 0; n < 8; ++n) acc4[k] = fmaf(sQ[32 * v + 8 * k + n], sLut[(ws[k] >> (4 * n)) & 15u], acc4[k]);
      }
      logit = ((acc4[0] + acc4[1]) + (acc4[2] + acc4[3])) * __half2float(ks[row]);
    }
    float gmax = logit;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, off));
    const float m_new = fmaxf(m_run, gmax);
    const float alpha = (m_run == -INFINITY) ? 0.0f : fast_exp2(m_run - m_new);
    const float p = (logit == -INFINITY) ? 0.0f : fast_exp2(logit - m_new);
    float psum = p;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
    l_run = l_run * alpha + psum;
    m_run = m_new;
#pragma unroll
    for (int k = 0; k < 4; ++k) o[k] *= alpha;
    const float pv = (t < seq_len) ? p * __half2float(vs[L.row(b, blk, min(t, seq_len - 1))]) : 0.0f;
    // The group's 32 value-code pairs of this lane's dims are all loaded before any is used
    // (one memory round trip per group); tokens past seq_len re-read the last token and get
    // weight 0.
    uint32_t two[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int ti = min(grp * 32 + i, seq_len - 1);
      two[i] = __ldg(reinterpret_cast<const uint16_t*>(vc + L.row(b, blk, ti) * 128 + half_off + 2 * lane));
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float pi = __shfl_sync(0xffffffffu, pv, i);
#pragma unroll
      for (int k = 0; k < 4; ++k) o[k] = fmaf(pi, sLut[(two[i] >> (4 * k)) & 15u], o[k]);
    }
  }
  if (lane == 0) {
    cm[warp] = m_run;
    cl[warp] = l_run;
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) co[warp][4 * lane + k] = o[k];
  __syncthreads();
  if (tid < kD) {
    float M = -INFINITY;
    for (int w = 0; w < kNf4DecWarps; ++w) M = fmaxf(M, cm[w]);
    float Ls = 0.0f, O = 0.0f;
    for (int w = 0; w < kNf4DecWarps; ++w) {
      const float wt = (cm[w] == -INFINITY) ? 0.0f : fast_exp2(cm[w] - M);
      Ls += cl[w] * wt;
      O += co[w][tid] * wt;
    }
    if (splits == 1) {
      out[static_cast<size_t>(bh) * kD + tid] = O / Ls;
    } else {
      const size_t pb = static_cast<size_t>(bh) * splits + split;
      part_o[pb * kD + tid] = O;
      if (tid == 0) {
        part_m[pb] = M;
        part_l[pb] = Ls;
      }
    }
  }
  if (splits == 1) return;
  // ticket after the barrier that follows this CTA's writes (acquire-release at GPU scope);
  // the last CTA folds the splits in eight at a time (one round trip to L2 per eight)
  __syncthreads();
  if (tid == 0) sLast = (ticket_add(&tickets[bh]) == static_cast<unsigned>(splits - 1));
  __syncthreads();
  if (!sLast) return;
  if (tid < kD) {
    const size_t p0 = static_cast<size_t>(bh) * splits;
    float M = -INFINITY, Ls = 0.0f, O = 0.0f;
    for (int s0 = 0; s0 < splits; s0 += 8) {
      float mv[8], lv[8], ov[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const bool in = s0 + u < splits;
        mv[u] = in ? __ldcg(part_m + p0 + s0 + u) : -INFINITY;
        lv[u] = in ? __ldcg(part_l + p0 + s0 + u) : 0.0f;
        ov[u] = in ? __ldcg(part_o + (p0 + s0 + u) * kD + tid) : 0.0f;
      }
      float mx = M;
#pragma unroll
      for (int u = 0; u < 8; ++u) mx = fmaxf(mx, mv[u]);
      if (mx == -INFINITY) continue;
      const float sc = (M == -INFINITY) ? 0.0f : fast_exp2(M - mx);
      Ls *= sc;
      O *= sc;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float wt = (mv[u] == -INFINITY) ? 0.0f : fast_exp2(mv[u] - mx);
        Ls += lv[u] * wt;
        O += ov[u] * wt;
      }
      M = mx;
    }
    out[static_cast<size_t>(bh) * kD + tid] = O / Ls;
  }
  if (tid == 0) tickets[bh] = 0u;
}

}  // namespace kvq
