// Quantize + pack: TQ-MSE-style scalar quantizer with Block-GTQ widths for K and a uniform
// width for V (page "RoPE-aware bit allocation for KV cache quantization", abstract: the
// allocator sits on TurboQuant-MSE, K and V get matched bit budgets, the cache is packed).
//
// One warp per 32-token tile of one (sequence, KV head) at a time (persistent warps);
// lane t quantizes token t of the tile. For a token row x (128 values):
//   s2   = sum_j x_j^2 in fp32, j ascending: fl32(s2 + fl32(x_j x_j))
//   norm = fp16(fp32 sqrt(s2)) (round to nearest even)
//   a    = fp32(sqrt(128)) / fp32(norm), 0 if norm == 0
//   y_j  = fp32(fp32(x_j a) g_b)            (V: g = 1, the multiply is skipped as exact)
//   code = #{thresholds of width w_b strictly below y_j}
// The code is found by binary search over the 2^w - 1 sorted thresholds, most significant
// bit first; the comparison at level p is bit p of the code, so its warp ballot (bit t =
// token t) is directly the tile's bit-plane word for that dim and plane.
// The tile is first copied into shared memory with a padded row pitch (65 words for 16-bit
// inputs), so that the 32 lanes reading the same dim of their own rows hit 32 banks.
// K: lane t works on token t. The ballot words are staged in shared memory and a last pass
//   turns each pair into the tile layout and writes whole lines. Per block b (ascending,
//   w_b > 0) and plane p, the ballots A (dim b) and B (dim b+64) give word0 = lo nibbles of
//   A's bytes | lo nibbles of B's bytes << 4 and word1 = hi nibbles of A | hi nibbles of B.
//   Bit s+4m of word H then holds token 4H + s + 8(m/2) at dim b (m even) or b+64 (m odd).
// V: lane l = c + 4m works on token 8(m/2) + 2c + (m%2), so a ballot is already the layout's
//   word (bit c+4m holds that token) and lane 0 stores each pair of words directly.
#pragma once

#include "common.cuh"

namespace kvq {

constexpr int kQuantWarps = 8;

template <int DT> struct QuantRow;
// 16-bit inputs: a row is 64 words (2 values each), pitch 65 words.
template <int DT> struct QuantRow16 {
  static constexpr int kPitch = kD / 2 + 1;
  static constexpr int kWords = kTile * kPitch;
  // Copy 32 rows (32 * 256 B, rows `row_stride` elements apart) into shared memory.
  __device__ __forceinline__ static void load(uint32_t* dst, const void* src, int64_t row_stride, int valid_rows,
                                              int lane) {
    const uint8_t* s8 = static_cast<const uint8_t*>(src);
    uint4 v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {             // all 16 loads in flight before any store
      const int idx = i * 32 + lane;           // 16-byte chunk of the tile
      const int r = idx >> 4, c = idx & 15;
      v[i] = make_uint4(0u, 0u, 0u, 0u);
      if (r < valid_rows) v[i] = __ldg(reinterpret_cast<const uint4*>(s8 + (static_cast<int64_t>(r) * row_stride * 2)) + c);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int idx = i * 32 + lane;
      const int r = idx >> 4, c = idx & 15;
      uint32_t* d = dst + r * kPitch + 4 * c;
      d[0] = v[i].x; d[1] = v[i].y; d[2] = v[i].z; d[3] = v[i].w;
    }
  }
  // Values 2i and 2i+1 of a row.
  __device__ __forceinline__ static float2 pair(const uint32_t* row, int i) {
    const uint32_t w = row[i];
    if constexpr (DT == KVQ_BF16) return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    else return __half22float2(*reinterpret_cast<const __half2*>(&w));
  }
};
template <> struct QuantRow<KVQ_BF16> : QuantRow16<KVQ_BF16> {};
template <> struct QuantRow<KVQ_F16> : QuantRow16<KVQ_F16> {};
// fp32 inputs: a row is 128 words, pitch 129 words.
template <> struct QuantRow<KVQ_F32> {
  static constexpr int kPitch = kD + 1;
  static constexpr int kWords = kTile * kPitch;
  __device__ __forceinline__ static void load(uint32_t* dst, const void* src, int64_t row_stride, int valid_rows,
                                              int lane) {
    const uint8_t* s8 = static_cast<const uint8_t*>(src);
#pragma unroll
    for (int h = 0; h < 2; ++h) {              // two batches of 16 loads in flight
      uint4 v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int idx = (16 * h + i) * 32 + lane;
        const int r = idx >> 5, c = idx & 31;
        v[i] = make_uint4(0u, 0u, 0u, 0u);
        if (r < valid_rows) v[i] = __ldg(reinterpret_cast<const uint4*>(s8 + (static_cast<int64_t>(r) * row_stride * 4)) + c);
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int idx = (16 * h + i) * 32 + lane;
        const int r = idx >> 5, c = idx & 31;
        uint32_t* d = dst + r * kPitch + 4 * c;
        d[0] = v[i].x; d[1] = v[i].y; d[2] = v[i].z; d[3] = v[i].w;
      }
    }
  }
  __device__ __forceinline__ static float2 pair(const uint32_t* row, int i) {
    return make_float2(__uint_as_float(row[2 * i]), __uint_as_float(row[2 * i + 1]));
  }
};

// fp16 norm of one row and the scale a = sqrt(128)/norm (0 for a zero norm).
template <int DT>
__device__ __forceinline__ void row_norm_scale(const uint32_t* row, __half& n16, float& a) {
  float s2 = 0.0f;
#pragma unroll 16
  for (int i = 0; i < kD / 2; ++i) {
    const float2 v = QuantRow<DT>::pair(row, i);
    s2 = __fadd_rn(s2, __fmul_rn(v.x, v.x));
    s2 = __fadd_rn(s2, __fmul_rn(v.y, v.y));
  }
  n16 = __float2half_rn(__fsqrt_rn(s2));
  const float nf = __half2float(n16);
  const float sqd = 11.313708305358887f;       // fp32(sqrt(128))
  a = (nf == 0.0f) ? 0.0f : __fdiv_rn(sqd, nf);
}

// Token handled by lane l in the values pass: l = c + 4m  ->  8(m/2) + 2c + (m%2).
__device__ __forceinline__ int value_token(int lane) { return 8 * (lane >> 3) + 2 * (lane & 3) + ((lane >> 2) & 1); }

// Binary search for two values of the same width W; the ballot of the comparison at level p
// (bit p of the code) is written by lane 0 to out[p * pstride] (first value) and
// out[p * pstride + 1] (second value). The top level compares with the middle threshold,
// which is exactly 0 for these symmetric codebooks. Widths up to 3 select the next
// threshold from registers (t[] holds the 2^W - 1 thresholds); wider ones index the
// shared-memory table.
template <int W>
__device__ __forceinline__ void search_ballot2(float y1, float y2, const float* __restrict__ thr, const float* t,
                                               uint32_t* out, int pstride, bool writer) {
  // out[p * pstride] and out[p * pstride + 1] are adjacent, 8-byte aligned words.
  auto put = [&](int p, bool c1, bool c2) {
    const unsigned A = __ballot_sync(0xffffffffu, c1);
    const unsigned B = __ballot_sync(0xffffffffu, c2);
    if (writer) *reinterpret_cast<uint2*>(out + p * pstride) = make_uint2(A, B);
  };
  const bool h1 = y1 > 0.0f, h2 = y2 > 0.0f;
  put(W - 1, h1, h2);
  if constexpr (W == 2) {
    put(0, y1 > (h1 ? t[2] : t[0]), y2 > (h2 ? t[2] : t[0]));
  } else if constexpr (W == 3) {
    const bool m1 = y1 > (h1 ? t[5] : t[1]), m2 = y2 > (h2 ? t[5] : t[1]);
    put(1, m1, m2);
    const float u1 = h1 ? (m1 ? t[6] : t[4]) : (m1 ? t[2] : t[0]);
    const float u2 = h2 ? (m2 ? t[6] : t[4]) : (m2 ? t[2] : t[0]);
    put(0, y1 > u1, y2 > u2);
  } else if constexpr (W >= 4) {
    int i1 = h1 ? (1 << (W - 1)) : 0, i2 = h2 ? (1 << (W - 1)) : 0;
#pragma unroll
    for (int p = W - 2; p >= 0; --p) {
      const int s = 1 << p;
      const bool c1 = y1 > thr[i1 + s - 1];
      const bool c2 = y2 > thr[i2 + s - 1];
      put(p, c1, c2);
      i1 += c1 ? s : 0;
      i2 += c2 ? s : 0;
    }
  }
}

// Dispatch on a runtime width (uniform across the warp).
__device__ __forceinline__ void search_ballot2_any(int w, float y1, float y2, const float* __restrict__ sThr,
                                                   const float* t3, uint32_t* out, int pstride, bool writer) {
  const float* thr = sThr + ((1 << w) - w - 1);
  switch (w) {
    case 1: search_ballot2<1>(y1, y2, thr, nullptr, out, pstride, writer); break;
    case 2: {
      const float t2[3] = {thr[0], thr[1], thr[2]};
      search_ballot2<2>(y1, y2, thr, t2, out, pstride, writer);
      break;
    }
    case 3: search_ballot2<3>(y1, y2, thr, t3, out, pstride, writer); break;
    case 4: search_ballot2<4>(y1, y2, thr, nullptr, out, pstride, writer); break;
    case 5: search_ballot2<5>(y1, y2, thr, nullptr, out, pstride, writer); break;
    case 6: search_ballot2<6>(y1, y2, thr, nullptr, out, pstride, writer); break;
    case 7: search_ballot2<7>(y1, y2, thr, nullptr, out, pstride, writer); break;
    default: search_ballot2<8>(y1, y2, thr, nullptr, out, pstride, writer); break;
  }
}

// Values: uniform width W for the whole row, dims processed in pairs.
template <int DT, int W>
__device__ __forceinline__ void quant_values(const uint32_t* myrow, float a, const float* __restrict__ sThr,
                                             uint32_t* vstage, bool writer) {
  const float* thr = sThr + ((1 << W) - W - 1);
  float t[7];
#pragma unroll
  for (int i = 0; i < 7; ++i) t[i] = (i < (1 << W) - 1) ? thr[i] : 0.0f;
#pragma unroll 4
  for (int i = 0; i < kD / 2; ++i) {
    const float2 x = QuantRow<DT>::pair(myrow, i);
    search_ballot2<W>(__fmul_rn(x.x, a), __fmul_rn(x.y, a), thr, t, vstage + 2 * i, kD, writer);
  }
}

template <int DT>
__global__ void __launch_bounds__(kQuantWarps * 32) kvq_quant_pack(
    const typename Elem<DT>::T* __restrict__ K, int64_t ksb, int64_t ksh, int64_t kst,
    const typename Elem<DT>::T* __restrict__ V, int64_t vsb, int64_t vsh, int64_t vst,
    int seq_len, int n_kv_heads, int tiles_written, int tiles_cap, const kvq_head_alloc* __restrict__ alloc,
    int bits_k, int bits_v, uint8_t* __restrict__ packed, int rec_bytes, long long n_tasks) {
  using Row = QuantRow<DT>;
  extern __shared__ __align__(16) uint32_t smem[];
  float* sThr = reinterpret_cast<float*>(smem);
  for (int i = threadIdx.x; i < kThresholdCount; i += blockDim.x) sThr[i] = c_tab.threshold[i];
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k_words = bits_k * kD, v_words = bits_v * kD;
  const int warp_words = Row::kWords + k_words + 2 * kH;
  uint32_t* rows = smem + 512 + warp * warp_words;
  uint32_t* stage = rows + Row::kWords;
  uint2* tb = reinterpret_cast<uint2*>(stage + k_words);   // per block: {gain bits, width | offset << 8}
  const uint32_t* myrow = rows + lane * Row::kPitch;
  const int vtok = value_token(lane);
  const uint32_t* myvrow = rows + vtok * Row::kPitch;
  const bool writer = lane == 0;
  float t3[7];
#pragma unroll
  for (int i = 0; i < 7; ++i) t3[i] = sThr[(1 << 3) - 3 - 1 + i];   // width-3 thresholds
  int cur_h = -1;

  for (long long task = static_cast<long long>(blockIdx.x) * kQuantWarps + warp; task < n_tasks;
       task += static_cast<long long>(gridDim.x) * kQuantWarps) {
    const int tile = static_cast<int>(task % tiles_written);
    const int bh = static_cast<int>(task / tiles_written);
    const int h = bh % n_kv_heads, b = bh / n_kv_heads;
    const kvq_head_alloc* al = alloc + h;
    if (al->k_words != k_words) continue;      // allocation made for another budget: write nothing
    if (h != cur_h) {
      __syncwarp();
      for (int i = lane; i < kH; i += 32)
        tb[i] = make_uint2(__float_as_uint(al->gain[i]), static_cast<uint32_t>(al->width[i]) |
                                                             (static_cast<uint32_t>(al->word_off[i]) << 8));
      cur_h = h;
    }
    const int t0 = tile * kTile;
    const int valid_rows = min(kTile, seq_len - t0);
    const bool valid = lane < valid_rows;

    // ---------------------------------------------------------------- K (Block-GTQ widths)
    __syncwarp();
    Row::load(rows, K + b * ksb + h * ksh + static_cast<int64_t>(t0) * kst, kst, valid_rows, lane);
    __syncwarp();
    __half kn16, vn16;
    float a;
    row_norm_scale<DT>(myrow, kn16, a);
    if (!valid) a = __int_as_float(0x7fc00000);   // NaN: every comparison false, so all code bits are 0
#pragma unroll 2
    for (int bp = 0; bp < kH / 2; ++bp) {
      const float2 lo = Row::pair(myrow, bp);             // dims 2bp, 2bp+1
      const float2 hi = Row::pair(myrow, kH / 2 + bp);    // dims 64+2bp, 65+2bp
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint2 e = tb[2 * bp + u];
        const int w = e.y & 0xffu;
        if (w == 0) continue;
        const float g = __uint_as_float(e.x);
        const float y1 = __fmul_rn(__fmul_rn(u ? lo.y : lo.x, a), g);
        const float y2 = __fmul_rn(__fmul_rn(u ? hi.y : hi.x, a), g);
        search_ballot2_any(w, y1, y2, sThr, t3, stage + (e.y >> 8), 2, writer);
      }
    }

    // ---------------------------------------------------------------- V (uniform width)
    uint8_t* rec = packed + (static_cast<size_t>(bh) * tiles_cap + tile) * rec_bytes;
    uint32_t* kout = reinterpret_cast<uint32_t*>(rec);
    uint32_t* vout = kout + k_words;
    const bool vvalid = vtok < valid_rows;
    __syncwarp();
    Row::load(rows, V + b * vsb + h * vsh + static_cast<int64_t>(t0) * vst, vst, valid_rows, lane);
    __syncwarp();
    row_norm_scale<DT>(myvrow, vn16, a);
    if (!vvalid) a = __int_as_float(0x7fc00000);
    switch (bits_v) {
      case 1: quant_values<DT, 1>(myvrow, a, sThr, vout, writer); break;
      case 2: quant_values<DT, 2>(myvrow, a, sThr, vout, writer); break;
      case 3: quant_values<DT, 3>(myvrow, a, sThr, vout, writer); break;
      case 4: quant_values<DT, 4>(myvrow, a, sThr, vout, writer); break;
      case 5: quant_values<DT, 5>(myvrow, a, sThr, vout, writer); break;
      case 6: quant_values<DT, 6>(myvrow, a, sThr, vout, writer); break;
      case 7: quant_values<DT, 7>(myvrow, a, sThr, vout, writer); break;
      default: quant_values<DT, 8>(myvrow, a, sThr, vout, writer); break;
    }
    __syncwarp();

    // ---------------------------------------------------------------- K words: permute + store
    for (int k = lane; k < k_words / 2; k += 32) {
      const uint32_t A = stage[2 * k], B = stage[2 * k + 1];
      uint2 o;
      o.x = (A & 0x0f0f0f0fu) | ((B & 0x0f0f0f0fu) << 4);
      o.y = ((A >> 4) & 0x0f0f0f0fu) | (B & 0xf0f0f0f0u);
      reinterpret_cast<uint2*>(kout)[k] = o;
    }
    uint16_t* norms = reinterpret_cast<uint16_t*>(vout + v_words);
    norms[lane] = valid ? __half_as_ushort(kn16) : 0;
    norms[kTile + vtok] = vvalid ? __half_as_ushort(vn16) : 0;
  }
}

// Dynamic shared memory of kvq_quant_pack for the input type's row pitch.
inline size_t quant_smem_bytes(int dtype, int bits_k, int bits_v) {
  const int row_words = (dtype == KVQ_F32) ? QuantRow<KVQ_F32>::kWords : QuantRow<KVQ_BF16>::kWords;
  return 4 * (512 + static_cast<size_t>(kQuantWarps) * (row_words + bits_k * kD + 2 * kH));
}

}  // namespace kvq
