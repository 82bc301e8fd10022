// Quantize + pack: TQ-MSE-style scalar quantizer with Block-GTQ widths for K and a uniform
// width for V (page "RoPE-aware bit allocation for KV cache quantization", abstract: the
// allocator sits on TurboQuant-MSE, K and V get matched bit budgets, the cache is packed).
//
// One warp per 32-token tile of one (sequence, KV head) at a time (persistent warps). For a
// token row x (128 values):
//   s2   = sum_j x_j^2 in fp32, j ascending: fl32(s2 + fl32(x_j x_j))
//   norm = fp16(fp32 sqrt(s2)) (round to nearest even)
//   a    = fp32(sqrt(128)) / fp32(norm), 0 if norm == 0
//   y_j  = fp32(fp32(x_j a) g_b)            (V: g = 1, the multiply is skipped as exact)
//   code = #{thresholds of width w_b strictly below y_j}
// The code is found by binary search over the 2^w - 1 sorted thresholds, most significant
// bit first. Tokens past the sequence length get a NaN scale, so every comparison is false
// and their codes are 0.
// The tile is first copied into shared memory with a padded row pitch (65 words for 16-bit
// inputs), so that 32 lanes reading one dim of their own rows hit 32 banks.
// K: lane t quantizes token t and appends its codes, in the allocation's stream order, to a
//   32-bit accumulator; the accumulator fills at the same code for every lane, so each full
//   word is one coalesced 128-byte warp store (word-planar tile layout).
// V: lane l quantizes dims 2l, 2l+1, 64+2l, 65+2l for the 32 tokens of the tile, placing
//   token t's code at bit bits_v * t of the dim's stream (positions known at compile time).
#pragma once

#include "common.cuh"

namespace kvq {

constexpr int kQuantWarps = 8;
constexpr int kQuantExtraWords = kTile + kH + kH / 4 + 8;   // per warp: 32 scales, 64 gains, 64 block indices, 8 classes

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
  // Value j of a row.
  __device__ __forceinline__ static float value(const uint32_t* row, int j) {
    const uint32_t w = row[j >> 1];
    const uint32_t u = (j & 1) ? (w >> 16) : (w & 0xffffu);
    if constexpr (DT == KVQ_BF16) return __uint_as_float(u << 16);
    else return __half2float(__ushort_as_half(static_cast<unsigned short>(u)));
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
  __device__ __forceinline__ static float value(const uint32_t* row, int j) { return __uint_as_float(row[j]); }
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

// Code of y for a width-W codebook: binary search, most significant bit first. The top
// level compares with the middle threshold, which is exactly 0 for these symmetric
// codebooks. Widths up to 3 select the next threshold from registers (t[] holds the
// 2^W - 1 thresholds); wider ones index the shared-memory table `thr`.
template <int W>
__device__ __forceinline__ uint32_t search_code(float y, const float* __restrict__ thr, const float* t) {
  const bool hi = y > 0.0f;
  if constexpr (W == 1) {
    return hi ? 1u : 0u;
  } else if constexpr (W == 2) {
    const bool lo = y > (hi ? t[2] : t[0]);
    return (hi ? 2u : 0u) | (lo ? 1u : 0u);
  } else if constexpr (W == 3) {
    const bool m = y > (hi ? t[5] : t[1]);
    const float u = hi ? (m ? t[6] : t[4]) : (m ? t[2] : t[0]);
    return (hi ? 4u : 0u) | (m ? 2u : 0u) | (y > u ? 1u : 0u);
  } else {
    int idx = hi ? (1 << (W - 1)) : 0;
#pragma unroll
    for (int p = W - 2; p >= 0; --p) {
      const int s = 1 << p;
      idx += (y > thr[idx + s - 1]) ? s : 0;
    }
    return static_cast<uint32_t>(idx);
  }
}

// Thresholds of width W from the shared table (all widths concatenated, width w at 2^w - w - 1).
__device__ __forceinline__ const float* width_thresholds(const float* sThr, int w) { return sThr + ((1 << w) - w - 1); }

// Bit stream writer for one lane's K codes; `fill` and `word` advance identically in every
// lane, so every flush is a full-warp store of one word-planar row (word i of 32 tokens).
struct KStream {
  uint32_t cur = 0;
  int fill = 0;
  int word = 0;
  template <int W>
  __device__ __forceinline__ void put(uint32_t code, uint32_t* __restrict__ kout, int lane) {
    cur |= code << fill;
    fill += W;
    if (fill >= 32) {
      kout[word * kTile + lane] = cur;
      ++word;
      fill -= 32;
      cur = fill ? (code >> (W - fill)) : 0u;
    }
  }
};

// All blocks of one width class: for each block b (stream order), the codes of dims b and
// b + 64. tb[b] = {gain bits of block b}; sb = the class's blocks.
template <int DT, int W>
__device__ __forceinline__ void quant_k_class(const uint32_t* myrow, float a, const float* __restrict__ gains,
                                              const uint8_t* __restrict__ sb, int nb, const float* __restrict__ sThr,
                                              KStream& ks, uint32_t* __restrict__ kout, int lane) {
  const float* thr = width_thresholds(sThr, W);
  float t[7];
#pragma unroll
  for (int i = 0; i < 7; ++i) t[i] = (W <= 3 && i < (1 << W) - 1) ? thr[i] : 0.0f;
  for (int k = 0; k < nb; ++k) {
    const int b = sb[k];
    const float g = gains[b];
    const float y1 = __fmul_rn(__fmul_rn(QuantRow<DT>::value(myrow, b), a), g);
    const float y2 = __fmul_rn(__fmul_rn(QuantRow<DT>::value(myrow, b + kH), a), g);
    ks.template put<W>(search_code<W>(y1, thr, t), kout, lane);
    ks.template put<W>(search_code<W>(y2, thr, t), kout, lane);
  }
}

// Values: width BV for every dim. Lane l handles dims {2l, 2l+1} and {64+2l, 65+2l}; sA[t]
// is token t's scale (NaN past the sequence length). Word i of dim j goes to vout[128 i + j].
template <int DT, int BV>
__device__ __forceinline__ void quant_v_tile(const uint32_t* rows, const float* sA, const float* __restrict__ sThr,
                                             uint32_t* __restrict__ vout, int lane) {
  const float* thr = width_thresholds(sThr, BV);
  float t[7];
#pragma unroll
  for (int i = 0; i < 7; ++i) t[i] = (BV <= 3 && i < (1 << BV) - 1) ? thr[i] : 0.0f;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int j0 = 2 * lane + kH * half;
    uint32_t w0[BV], w1[BV];
#pragma unroll
    for (int i = 0; i < BV; ++i) { w0[i] = 0u; w1[i] = 0u; }
#pragma unroll
    for (int tok = 0; tok < kTile; ++tok) {
      const float2 x = QuantRow<DT>::pair(rows + tok * QuantRow<DT>::kPitch, j0 >> 1);
      const float at = sA[tok];
      const uint32_t c0 = search_code<BV>(__fmul_rn(x.x, at), thr, t);
      const uint32_t c1 = search_code<BV>(__fmul_rn(x.y, at), thr, t);
      const int bit = BV * tok, wi = bit >> 5, sh = bit & 31;
      w0[wi] |= c0 << sh;
      w1[wi] |= c1 << sh;
      if (sh + BV > 32) {
        w0[wi + 1] |= c0 >> (32 - sh);
        w1[wi + 1] |= c1 >> (32 - sh);
      }
    }
#pragma unroll
    for (int i = 0; i < BV; ++i)
      *reinterpret_cast<uint2*>(vout + i * kD + j0) = make_uint2(w0[i], w1[i]);
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
  const int k_words = bits_k * kD;
  uint32_t* wbase = smem + 512 + warp * (Row::kWords + kQuantExtraWords);
  uint32_t* rows = wbase;
  float* sA = reinterpret_cast<float*>(wbase + Row::kWords);             // 32 value scales
  float* sGain = sA + kTile;                                              // 64 block gains
  uint8_t* sBlk = reinterpret_cast<uint8_t*>(sGain + kH);                 // 64 blocks, stream order
  const uint32_t* myrow = rows + lane * Row::kPitch;
  uint32_t* sCls = reinterpret_cast<uint32_t*>(sBlk + kH);              // 8 classes: width | first << 8 | blocks << 16
  int cur_h = -1, n_cls = 0;

  for (long long task = static_cast<long long>(blockIdx.x) * kQuantWarps + warp; task < n_tasks;
       task += static_cast<long long>(gridDim.x) * kQuantWarps) {
    const int tile = static_cast<int>(task % tiles_written);
    const int bh = static_cast<int>(task / tiles_written);
    const int h = bh % n_kv_heads, b = bh / n_kv_heads;
    const kvq_head_alloc* al = alloc + h;
    if (al->k_words != k_words) continue;      // allocation made for another budget: write nothing
    if (h != cur_h) {
      __syncwarp();
      for (int i = lane; i < kH; i += 32) {
        sGain[i] = al->gain[i];
        sBlk[i] = al->stream_block[i];
      }
      n_cls = min(max(al->n_classes, 0), 8);
      if (lane < 8)
        sCls[lane] = static_cast<uint32_t>(al->class_width[lane]) | (static_cast<uint32_t>(al->class_first[lane]) << 8) |
                     (static_cast<uint32_t>(al->class_blocks[lane]) << 16);
      __syncwarp();
      cur_h = h;
    }
    const int t0 = tile * kTile;
    const int valid_rows = min(kTile, seq_len - t0);
    const bool valid = lane < valid_rows;
    uint8_t* rec = packed + (static_cast<size_t>(bh) * tiles_cap + tile) * rec_bytes;
    uint32_t* kout = reinterpret_cast<uint32_t*>(rec);
    uint16_t* norms = reinterpret_cast<uint16_t*>(kout + k_words);   // 32 K norms, then 32 V norms
    uint32_t* vout = kout + k_words + kTile;

    // ---------------------------------------------------------------- K (Block-GTQ widths)
    __syncwarp();
    Row::load(rows, K + b * ksb + h * ksh + static_cast<int64_t>(t0) * kst, kst, valid_rows, lane);
    __syncwarp();
    __half n16;
    float a;
    row_norm_scale<DT>(myrow, n16, a);
    norms[lane] = valid ? __half_as_ushort(n16) : 0;
    if (!valid) a = __int_as_float(0x7fc00000);   // NaN: every comparison false, so all codes are 0
    KStream ks;
    for (int c = 0; c < n_cls; ++c) {
      const uint32_t e = sCls[c];
      const int w = e & 0xffu, first = (e >> 8) & 0xffu, nb = e >> 16;
      const uint8_t* sb = sBlk + first;
      switch (w) {
        case 1: quant_k_class<DT, 1>(myrow, a, sGain, sb, nb, sThr, ks, kout, lane); break;
        case 2: quant_k_class<DT, 2>(myrow, a, sGain, sb, nb, sThr, ks, kout, lane); break;
        case 3: quant_k_class<DT, 3>(myrow, a, sGain, sb, nb, sThr, ks, kout, lane); break;
        case 4: quant_k_class<DT, 4>(myrow, a, sGain, sb, nb, sThr, ks, kout, lane); break;
        case 5: quant_k_class<DT, 5>(myrow, a, sGain, sb, nb, sThr, ks, kout, lane); break;
        case 6: quant_k_class<DT, 6>(myrow, a, sGain, sb, nb, sThr, ks, kout, lane); break;
        case 7: quant_k_class<DT, 7>(myrow, a, sGain, sb, nb, sThr, ks, kout, lane); break;
        default: quant_k_class<DT, 8>(myrow, a, sGain, sb, nb, sThr, ks, kout, lane); break;
      }
    }

    // ---------------------------------------------------------------- V (uniform width)
    __syncwarp();
    Row::load(rows, V + b * vsb + h * vsh + static_cast<int64_t>(t0) * vst, vst, valid_rows, lane);
    __syncwarp();
    row_norm_scale<DT>(myrow, n16, a);
    norms[kTile + lane] = valid ? __half_as_ushort(n16) : 0;
    sA[lane] = valid ? a : __int_as_float(0x7fc00000);
    __syncwarp();
    switch (bits_v) {
      case 1: quant_v_tile<DT, 1>(rows, sA, sThr, vout, lane); break;
      case 2: quant_v_tile<DT, 2>(rows, sA, sThr, vout, lane); break;
      case 3: quant_v_tile<DT, 3>(rows, sA, sThr, vout, lane); break;
      case 4: quant_v_tile<DT, 4>(rows, sA, sThr, vout, lane); break;
      case 5: quant_v_tile<DT, 5>(rows, sA, sThr, vout, lane); break;
      case 6: quant_v_tile<DT, 6>(rows, sA, sThr, vout, lane); break;
      case 7: quant_v_tile<DT, 7>(rows, sA, sThr, vout, lane); break;
      default: quant_v_tile<DT, 8>(rows, sA, sThr, vout, lane); break;
    }
  }
}

// Dynamic shared memory of kvq_quant_pack: thresholds + per warp the row tile, 32 value
// scales, 64 gains, 64 stream-order block indices and the 8-entry class table.
inline size_t quant_smem_bytes(int dtype) {
  const int row_words = (dtype == KVQ_F32) ? QuantRow<KVQ_F32>::kWords : QuantRow<KVQ_BF16>::kWords;
  return 4 * (512 + static_cast<size_t>(kQuantWarps) * (row_words + kQuantExtraWords));
}

}  // namespace kvq
