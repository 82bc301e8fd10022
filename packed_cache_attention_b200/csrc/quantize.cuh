// Quantize + pack: TQ-MSE-style scalar quantizer with Block-GTQ widths for K and a uniform
// width for V ("RoPE-aware bit allocation for KV cache quantization", abstract: Block-GTQ
// is "built on TurboQuant-MSE", "matched K/V bit budgets", "packed K3V3").
//
// One warp per 32-token tile of one (sequence, KV head); lane t quantizes token t of the
// tile. For a token row x (128 values):
//   s2   = sum_j x_j^2 in fp64, j ascending (exact products, rounded sums)
//   norm = fp16(sqrt(s2)) (round to nearest even)
//   a    = fp32(sqrt(128)) / fp32(norm), 0 if norm == 0
//   y_j  = fp32(fp32(x_j a) g_b)            (V: g = 1, the multiply is skipped as exact)
//   code = #{thresholds of width w_b strictly below y_j}  (branch-free binary search)
// Bit planes are gathered with warp ballots (bit t = token t) and staged in shared memory;
// a last pass permutes them into the tile layout and writes whole 128-byte lines:
//   K, per block b (ascending, w_b > 0), per plane p: two words built from the ballots
//      A (dim b) and B (dim b+64): word0 = lo nibbles of A's bytes | lo nibbles of B's bytes
//      << 4, word1 = hi nibbles of A | hi nibbles of B. Bit s+4m of word H then holds token
//      4H + s + 8(m/2) at dim b (m even) or b+64 (m odd).
//   V, per plane p, per dim j: the ballot word with each byte's bits unzipped (even bits
//      to the low nibble, odd bits to the high nibble): bit c+4m holds token
//      8(m/2) + 2c + (m%2).
#pragma once

#include "common.cuh"

namespace kvq {

constexpr int kQuantWarps = 8;

// Row of 128 stored values of one token, held in registers.
template <int DT> struct RowRegs;
template <> struct RowRegs<KVQ_F32> {
  float r[kD];
  __device__ __forceinline__ void load(const float* p) {
#pragma unroll
    for (int i = 0; i < kD / 4; ++i) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(p) + i);
      r[4 * i] = v.x; r[4 * i + 1] = v.y; r[4 * i + 2] = v.z; r[4 * i + 3] = v.w;
    }
  }
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int i = 0; i < kD; ++i) r[i] = 0.0f;
  }
  __device__ __forceinline__ float get(int j) const { return r[j]; }
};
template <int DT> struct RowRegs16 {
  uint32_t r[kD / 2];
  __device__ __forceinline__ void load(const void* p) {
#pragma unroll
    for (int i = 0; i < kD / 8; ++i) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(p) + i);
      r[4 * i] = v.x; r[4 * i + 1] = v.y; r[4 * i + 2] = v.z; r[4 * i + 3] = v.w;
    }
  }
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int i = 0; i < kD / 2; ++i) r[i] = 0u;
  }
  __device__ __forceinline__ float get(int j) const {
    const uint32_t bits = (j & 1) ? (r[j >> 1] >> 16) : (r[j >> 1] & 0xffffu);
    if constexpr (DT == KVQ_BF16) return __uint_as_float(bits << 16);
    else return __half2float(__ushort_as_half(static_cast<unsigned short>(bits)));
  }
};
template <> struct RowRegs<KVQ_F16> : RowRegs16<KVQ_F16> {};
template <> struct RowRegs<KVQ_BF16> : RowRegs16<KVQ_BF16> {};

// code = #{t in thresholds(w) : t < y} by branch-free binary search over the 2^w - 1
// sorted thresholds (shared-memory copy of the constant table).
__device__ __forceinline__ int lm_code(float y, int w, const float* __restrict__ sThr) {
  const float* t = sThr + ((1 << w) - w - 1);
  int idx = 0;
#pragma unroll
  for (int k = 7; k >= 0; --k) {
    if (k < w) {
      const int s = 1 << k;
      idx += (y > t[idx + s - 1]) ? s : 0;
    }
  }
  return idx;
}

// fp16 norm and scale of a row, as in the header comment.
template <int DT>
__device__ __forceinline__ void row_norm_scale(const RowRegs<DT>& row, __half& n16, float& a) {
  double s2 = 0.0;
#pragma unroll
  for (int j = 0; j < kD; ++j) {
    const double x = static_cast<double>(row.get(j));
    s2 = __fma_rn(x, x, s2);        // x*x is exact in fp64, so this is fl(s2 + x^2)
  }
  n16 = __double2half(__dsqrt_rn(s2));
  const float nf = __half2float(n16);
  const float sqd = 11.313708305358887f;       // fp32(sqrt(128))
  a = (nf == 0.0f) ? 0.0f : __fdiv_rn(sqd, nf);
}

__device__ __forceinline__ uint32_t unzip_bytes(uint32_t x) {
  uint32_t t = (x ^ (x >> 1)) & 0x22222222u;
  x ^= t ^ (t << 1);
  t = (x ^ (x >> 2)) & 0x0c0c0c0cu;
  x ^= t ^ (t << 2);
  return x;
}

template <int DT>
__global__ void __launch_bounds__(kQuantWarps * 32) kvq_quant_pack(
    const typename Elem<DT>::T* __restrict__ K, int64_t ksb, int64_t ksh, int64_t kst,
    const typename Elem<DT>::T* __restrict__ V, int64_t vsb, int64_t vsh, int64_t vst,
    int seq_len, int n_kv_heads, int tiles_written, int tiles_cap, const kvq_head_alloc* __restrict__ alloc,
    int bits_k, int bits_v, uint8_t* __restrict__ packed, int rec_bytes, long long n_tasks) {
  extern __shared__ __align__(16) uint32_t smem[];
  float* sThr = reinterpret_cast<float*>(smem);
  for (int i = threadIdx.x; i < kThresholdCount; i += blockDim.x) sThr[i] = c_tab.threshold[i];
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long task = static_cast<long long>(blockIdx.x) * kQuantWarps + warp;
  if (task >= n_tasks) return;
  const int k_words = bits_k * kD, v_words = bits_v * kD;
  uint32_t* stage = smem + 512 + warp * (k_words + v_words);
  uint32_t* vstage = stage + k_words;

  const int tile = static_cast<int>(task % tiles_written);
  const int bh = static_cast<int>(task / tiles_written);
  const int h = bh % n_kv_heads, b = bh / n_kv_heads;
  const kvq_head_alloc* al = alloc + h;
  if (al->k_words != k_words) return;        // allocation made for another budget: write nothing
  const int token = tile * kTile + lane;
  const bool valid = token < seq_len;

  RowRegs<DT> row;
  __half kn16, vn16;
  float a;

  // ---------------------------------------------------------------- K (Block-GTQ widths)
  if (valid) row.load(K + b * ksb + h * ksh + static_cast<int64_t>(token) * kst);
  else row.zero();
  row_norm_scale<DT>(row, kn16, a);
#pragma unroll
  for (int blk = 0; blk < kH; ++blk) {
    const int w = al->width[blk];
    if (w == 0) continue;
    const float g = al->gain[blk];
    const float y1 = __fmul_rn(__fmul_rn(row.get(blk), a), g);
    const float y2 = __fmul_rn(__fmul_rn(row.get(blk + kH), a), g);
    const int c1 = lm_code(y1, w, sThr);
    const int c2 = lm_code(y2, w, sThr);
    uint32_t* dst = stage + al->word_off[blk];
    for (int p = 0; p < w; ++p) {
      const unsigned A = __ballot_sync(0xffffffffu, valid && ((c1 >> p) & 1));
      const unsigned B = __ballot_sync(0xffffffffu, valid && ((c2 >> p) & 1));
      if (lane == 0) {
        dst[2 * p] = A;
        dst[2 * p + 1] = B;
      }
    }
  }

  // ---------------------------------------------------------------- V (uniform width)
  if (valid) row.load(V + b * vsb + h * vsh + static_cast<int64_t>(token) * vst);
  else row.zero();
  row_norm_scale<DT>(row, vn16, a);
#pragma unroll
  for (int j = 0; j < kD; ++j) {
    const float y = __fmul_rn(row.get(j), a);
    const int c = lm_code(y, bits_v, sThr);
    for (int p = 0; p < bits_v; ++p) {
      const unsigned W = __ballot_sync(0xffffffffu, valid && ((c >> p) & 1));
      if (lane == 0) vstage[p * kD + j] = W;
    }
  }
  __syncwarp();

  // ---------------------------------------------------------------- permute + store
  uint8_t* rec = packed + (static_cast<size_t>(bh) * tiles_cap + tile) * rec_bytes;
  uint32_t* kout = reinterpret_cast<uint32_t*>(rec);
  for (int k = lane; k < k_words / 2; k += 32) {
    const uint32_t A = stage[2 * k], B = stage[2 * k + 1];
    uint2 o;
    o.x = (A & 0x0f0f0f0fu) | ((B & 0x0f0f0f0fu) << 4);
    o.y = ((A >> 4) & 0x0f0f0f0fu) | (B & 0xf0f0f0f0u);
    reinterpret_cast<uint2*>(kout)[k] = o;
  }
  uint32_t* vout = kout + k_words;
  for (int k = lane; k < v_words; k += 32) vout[k] = unzip_bytes(vstage[k]);
  uint16_t* norms = reinterpret_cast<uint16_t*>(vout + v_words);
  norms[lane] = valid ? __half_as_ushort(kn16) : 0;
  norms[kTile + lane] = valid ? __half_as_ushort(vn16) : 0;
}

}  // namespace kvq
