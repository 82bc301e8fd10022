// Calibration kernels: the label-free energy score per RoPE block and the greedy integer
// bit allocation by marginal gain, computed per layer and KV head (page "RoPE-aware bit
// allocation for KV cache quantization", abstract).
#pragma once

#include <type_traits>

#include "common.cuh"

namespace kvq {

// Non-coherent global loads issued as volatile asm, so all loads of a batch are issued
// before the arithmetic that consumes them (keeps many rows in flight per lane).
template <typename V> __device__ __forceinline__ V ldg_stream(const void* p);
template <> __device__ __forceinline__ uint2 ldg_stream<uint2>(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];\n" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
template <> __device__ __forceinline__ float4 ldg_stream<float4>(const void* p) {
  float4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];\n"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

constexpr int kCalibSegment = 64;      // chunk sums per fixed-order segment sum
#ifndef KVQ_CALIB_CHUNKS_PER_CTA
#define KVQ_CALIB_CHUNKS_PER_CTA 4
#endif
// 16 lanes per chunk; 4 chunks (64 threads) per CTA give about 7 resident CTAs on every SM at
// 128K tokens, so the single wave is evenly loaded. It must divide kCalibSegment.
constexpr int kCalibChunksPerCta = KVQ_CALIB_CHUNKS_PER_CTA;
static_assert(64 % kCalibChunksPerCta == 0, "a CTA's chunks lie in one segment");

// Calibration workspace after the status header: per KV head a head counter and one counter
// per segment (unsigned, zero between calls), then energies E[h][64], segment sums
// [h][n_seg][64] and chunk sums [h][n_chunks][64] (fp64).
struct CalibWs {
  unsigned* head_count;   // [H]
  unsigned* seg_count;    // [H][n_seg]
  double* energy;         // [H][64]
  double* seg_sum;        // [H][n_seg][64]
  double* chunk_sum;      // [H][n_chunks][64]
};

// Grid (ceil(n_chunks / kCalibChunksPerCta), n_kv_heads), 16 lanes per 64-token chunk. Lane k
// (0..15) of a chunk owns blocks 4k..4k+3, i.e. dims 4k..4k+3 and 64+4k..67+4k, read as two
// 4-element vectors per token (128 contiguous bytes per half-warp for 16-bit inputs). Within
// the chunk the pooled tokens u = s*n_calib + t are summed left to right in fp64, each term
// being fl(fl(x^2) + fl(y^2)).
// The CTA that completes a segment (atomic ticket per segment) sums that segment's 64 chunk
// sums left to right; the CTA that completes the last segment of a head sums the segment
// sums left to right and writes E_b = total / N. Counters are reset to zero for the next call.
template <int DT>
__global__ void __launch_bounds__(16 * kCalibChunksPerCta, 32 / kCalibChunksPerCta) kvq_calib_reduce(
    const typename Elem<DT>::T* __restrict__ K, int n_calib, int64_t sb, int64_t sh, int64_t st, int N,
    int n_chunks, CalibWs ws) {
  using T = typename Elem<DT>::T;
  __shared__ int sTicket;
  const int h = blockIdx.y;
  const int chunk = blockIdx.x * kCalibChunksPerCta + (threadIdx.x >> 4);
  const int k = threadIdx.x & 15;
  const int n_seg = (n_chunks + kCalibSegment - 1) / kCalibSegment;
  grid_dependency_wait();                                   // K and the counters may be the previous kernel's
  if (chunk < n_chunks) {
    const int u0 = chunk * kCalibChunk;
    const int n = min(N - u0, kCalibChunk);
    int s = u0 / n_calib;
    int t = u0 - s * n_calib;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    // acc_j += fl(fl(x_j^2) + fl(y_j^2)) for the 4 dims x (blocks 4k..4k+3) and their partners y
    auto add_vals = [&](const auto& a, const auto& b) {
      float x[4], y[4];
      if constexpr (DT == KVQ_F32) {
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        y[0] = b.x; y[1] = b.y; y[2] = b.z; y[3] = b.w;
      } else {
        const uint32_t av[2] = {a.x, a.y}, bv[2] = {b.x, b.y};
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          x[2 * j] = Elem<DT>::to_f32(bits_to<T>(av[j] & 0xffffu));
          x[2 * j + 1] = Elem<DT>::to_f32(bits_to<T>(av[j] >> 16));
          y[2 * j] = Elem<DT>::to_f32(bits_to<T>(bv[j] & 0xffffu));
          y[2 * j + 1] = Elem<DT>::to_f32(bits_to<T>(bv[j] >> 16));
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const double dx = x[j], dy = y[j];
        acc[j] = __dadd_rn(acc[j], __dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy)));
      }
    };
    auto add_row = [&](const T* row) {
      using V2 = typename std::conditional<DT == KVQ_F32, float4, uint2>::type;
      add_vals(__ldg(reinterpret_cast<const V2*>(row + 4 * k)), __ldg(reinterpret_cast<const V2*>(row + kH + 4 * k)));
    };
    if (n == kCalibChunk && t + kCalibChunk <= n_calib) {
      // whole chunk inside one sequence: 16 rows of loads in flight before any arithmetic
      const T* base = K + s * sb + h * sh + static_cast<int64_t>(t) * st;
#pragma unroll 1
      for (int i0 = 0; i0 < kCalibChunk; i0 += 16) {
        using V2 = typename std::conditional<DT == KVQ_F32, float4, uint2>::type;
        V2 va[16], vb[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const T* row = base + static_cast<int64_t>(i0 + i) * st;
          va[i] = ldg_stream<V2>(row + 4 * k);
          vb[i] = ldg_stream<V2>(row + kH + 4 * k);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) add_vals(va[i], vb[i]);
      }
    } else {
      for (int i = 0; i < n; ++i) {
        add_row(K + s * sb + h * sh + static_cast<int64_t>(t) * st);
        if (++t == n_calib) {
          t = 0;
          ++s;
        }
      }
    }
    double* dst = ws.chunk_sum + (static_cast<size_t>(h) * n_chunks + chunk) * kH + 4 * k;
#pragma unroll
    for (int j = 0; j < 4; ++j) dst[j] = acc[j];
  }

  // ---- segment completion (chunks of one CTA always lie in one segment: 8 divides 64)
  const int seg = (blockIdx.x * kCalibChunksPerCta) / kCalibSegment;
  const int c0 = seg * kCalibSegment, c1 = min(n_chunks, c0 + kCalibSegment);
  const int mine = min(n_chunks, (blockIdx.x + 1) * kCalibChunksPerCta) - blockIdx.x * kCalibChunksPerCta;
  allow_dependents();
  // tickets are taken after the barrier that follows the writes they publish, with
  // acquire-release order at GPU scope (no separate fences)
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned* cnt = ws.seg_count + static_cast<size_t>(h) * n_seg + seg;
    const unsigned done = ticket_add(cnt, static_cast<unsigned>(mine)) + mine;
    sTicket = (done == static_cast<unsigned>(c1 - c0));
    if (sTicket) *cnt = 0u;
  }
  __syncthreads();
  if (!sTicket) return;
  if (threadIdx.x < kH) {
    const double* src = ws.chunk_sum + (static_cast<size_t>(h) * n_chunks) * kH + threadIdx.x;
    double acc = 0.0;
#pragma unroll 32
    for (int c = c0; c < c1; ++c) acc = __dadd_rn(acc, __ldcg(src + static_cast<size_t>(c) * kH));
    ws.seg_sum[(static_cast<size_t>(h) * n_seg + seg) * kH + threadIdx.x] = acc;
  }
  // ---- head completion
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned done = ticket_add(ws.head_count + h) + 1u;
    sTicket = (done == static_cast<unsigned>(n_seg));
    if (sTicket) ws.head_count[h] = 0u;
  }
  __syncthreads();
  if (!sTicket) return;
  if (threadIdx.x < kH) {
    const double* src = ws.seg_sum + static_cast<size_t>(h) * n_seg * kH + threadIdx.x;
    double S = 0.0;
#pragma unroll 8
    for (int g = 0; g < n_seg; ++g) S = __dadd_rn(S, __ldcg(src + static_cast<size_t>(g) * kH));
    ws.energy[static_cast<size_t>(h) * kH + threadIdx.x] = __ddiv_rn(S, static_cast<double>(N));
  }
}

// One CTA of 512 threads per KV head, after kvq_calib_reduce has written E[h][64].
//  1. Greedy allocation in rank form: entry e = 8b + w (w < w_max) has marginal gain
//     E_b (delta(w) - delta(w+1)); the greedy takes the bits_k * 64 first entries in the
//     order (gain descending, e ascending). Because delta is strictly convex each block's
//     gains are non-increasing in w, so this is the step-by-step greedy with ties to the
//     lowest block, the entries of a block that precede a given entry form a prefix (found
//     by binary search), and the picked entries of a block are a prefix: w_b = their count.
//  2. g_b, f_b, the K stream order and bit offsets, the decode plan (width classes cut into
//     slots of 4 block pairs) and the allocation digest.
// The record is built in shared memory and copied out whole at the end.
__global__ void __launch_bounds__(512) kvq_greedy_alloc(const double* __restrict__ energy, int bits_k, int w_max,
                                                        int mode, kvq_head_alloc* __restrict__ alloc) {
  static_assert(sizeof(kvq_head_alloc) % 16 == 0 && sizeof(kvq_head_alloc) <= 512 * 16, "record copy");
  __shared__ double sE[kH];
  __shared__ long long sKey[kH * 8];
  __shared__ short sIdx[kH * 8];
  __shared__ int sWidth[kH];
  __shared__ int sCount[9];
  __shared__ int sClsX0[9];
  __shared__ uint64_t sDig[2];
  __shared__ double sSum;
  __shared__ __align__(16) kvq_head_alloc sRec;
  const int h = blockIdx.x, tid = threadIdx.x;
  kvq_head_alloc* al = &sRec;
  uint32_t* rec_words = reinterpret_cast<uint32_t*>(&sRec);
  constexpr int kRecWords = static_cast<int>(sizeof(kvq_head_alloc) / 4);
  for (int i = tid; i < kRecWords; i += blockDim.x) rec_words[i] = 0u;
  grid_dependency_wait();                                   // the energies come from the reduction
  if (tid < kH) sE[tid] = __ldcg(energy + static_cast<size_t>(h) * kH + tid);
  __syncthreads();
  if (tid == 0) {
    double S = 0.0;
    for (int b = 0; b < kH; ++b) S = __dadd_rn(S, sE[b]);
    sSum = S;
  }
  {
    const int b = tid >> 3, w = tid & 7;
    const bool valid = w < w_max;
    const double gv = valid ? __dmul_rn(sE[b], __dsub_rn(static_cast<double>(c_tab.delta[w]),
                                                          static_cast<double>(c_tab.delta[w + 1])))
                            : -1.0;
    // valid gains are >= 0 (+0 for a zero energy); invalid entries never precede a valid one
    sKey[tid] = valid ? __double_as_longlong(gv) : -1LL;
    sIdx[tid] = static_cast<short>(tid);
    if (tid < kH) sWidth[tid] = 0;
  }
  __syncthreads();
  if (mode == KVQ_MODE_UNIFORM) {
    if (tid < kH) sWidth[tid] = bits_k;
  } else {
    // Sort the 512 entries by (gain descending, entry ascending) with a bitonic network;
    // the first bits_k * 64 are the greedy's picks. Non-negative doubles order like their
    // bit patterns, so keys are 64-bit integers; entries at or above w_max get key -1 and
    // sort after every valid one.
    // Compare-exchange distances of 32 and more go through shared memory, shorter ones
    // between the lanes of a warp (thread tid holds entry tid in registers there).
    // A block's 8 entries are already in order (its gains do not increase with w, and equal
    // keys are ordered by entry), so the network starts at runs of 16: runs of 8 must be in
    // order where (position & 8) == 0 and reversed elsewhere, so odd blocks are read reversed.
    const int src = (tid & 8) ? (tid ^ 7) : tid;
    long long key = sKey[src];
    int idx = sIdx[src];
    for (int k = 16; k <= kH * 8; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        if (j >= 32) {
          sKey[tid] = key;
          sIdx[tid] = static_cast<short>(idx);
          __syncthreads();
          const long long ko = sKey[tid ^ j];
          const int io = sIdx[tid ^ j];
          __syncthreads();
          const bool lower = (tid & j) == 0;                     // this thread holds the pair's first slot
          const bool up = (tid & k) == 0;                        // the pair's block sorts descending-first
          const bool mine_first = (key > ko) || (key == ko && idx < io);
          if (mine_first != (lower == up)) { key = ko; idx = io; }
        } else {
          const long long ko = __shfl_xor_sync(0xffffffffu, key, j);
          const int io = __shfl_xor_sync(0xffffffffu, idx, j);
          const bool lower = (tid & j) == 0;
          const bool up = (tid & k) == 0;
          const bool mine_first = (key > ko) || (key == ko && idx < io);
          if (mine_first != (lower == up)) { key = ko; idx = io; }
        }
      }
    }
    if (tid < bits_k * kH) atomicAdd(&sWidth[idx >> 3], 1);
  }
  if (tid < 9) sCount[tid] = 0;
  __syncthreads();

  if (tid < kH) {
    const int b = tid;
    float g = 1.0f;
    if (mode != KVQ_MODE_UNIFORM && sE[b] > 0.0 && sSum > 0.0)
      g = __double2float_rn(__dsqrt_rn(__ddiv_rn(__dmul_rn(2.0, sSum), __dmul_rn(static_cast<double>(kD), sE[b]))));
    al->energy[b] = sE[b];
    al->gain[b] = g;
    al->dequant[b] = __double2float_rn(__ddiv_rn(1.0, __dmul_rn(__dsqrt_rn(static_cast<double>(kD)),
                                                                static_cast<double>(g))));
    const int w = sWidth[b];
    al->width[b] = static_cast<uint8_t>(w);
    atomicAdd(&sCount[w], 1);
    // Stream order: width classes 8..1, blocks ascending inside a class; each block is a
    // pair of codes (dim b, dim b + 64) of w_b bits each. Block b's position and bit offset
    // count the wider blocks and the lower blocks of its own width.
    int pos = 0, bit = 0;
    for (int c = 0; c < kH; ++c) {
      const int wc = sWidth[c];
      if (wc > w || (wc == w && c < b)) {
        ++pos;
        bit += 2 * wc;
      }
    }
    if (w > 0) {
      al->stream_block[pos] = static_cast<uint8_t>(b);
      al->bit_off[b] = static_cast<int16_t>(bit);
    } else {
      al->bit_off[b] = -1;
    }
  }
  __syncthreads();
  // Class table (stream order: widths 8..1) and, per class, its first group of the decode plan.
  if (tid == 0) {
    int pos = 0, bit = 0, n_cls = 0, x0 = 0;
    for (int w = 8; w >= 1; --w) {
      const int nb = sCount[w];
      if (nb == 0) continue;
      al->class_width[n_cls] = static_cast<uint8_t>(w);
      al->class_first[n_cls] = static_cast<uint8_t>(pos);
      al->class_blocks[n_cls] = static_cast<uint8_t>(nb);
      al->class_bit[n_cls] = static_cast<uint16_t>(bit);
      sClsX0[n_cls] = x0;
      x0 += (nb + 3) >> 2;
      pos += nb;
      bit += 2 * w * nb;
      ++n_cls;
    }
    for (int c = n_cls; c < 8; ++c) {
      al->class_width[c] = 0;
      al->class_first[c] = static_cast<uint8_t>(pos);
      al->class_blocks[c] = 0;
      al->class_bit[c] = static_cast<uint16_t>(bit);
      sClsX0[c] = x0;
    }
    sClsX0[8] = x0;
    al->n_classes = n_cls;
    al->n_blocks = pos;
    al->k_words = bit / 32 * kTile;     // bits per token * 32 tokens / 32 bits per word
    al->head_dim = kD;
    al->bits_k = bits_k;
    al->w_max = w_max;
    al->mode = mode;
    al->reserved = 0;
  }
  if (tid < kH && tid >= kH - sCount[0]) al->stream_block[tid] = 0xffu;   // positions past the last block
  if (tid < 96) al->plan_col_block[tid] = -1;
  __syncthreads();
  // Decode plan: classes in stream order cut into slots of 4 consecutive block pairs (a
  // class's last slot holds what is left); slot s covers columns 4s .. 4s + 3. One thread per
  // slot; slots of a class start at that class's first slot index sClsX0[c].
  const int n_slots = sClsX0[8];
  if (tid < n_slots) {
    const int x = tid;
    int c = 0;
    while (sClsX0[c + 1] <= x) ++c;
    const int w = al->class_width[c], nb = al->class_blocks[c], first = al->class_first[c];
    const int k = x - sClsX0[c];
    al->plan_slot[x] = static_cast<uint32_t>(w) | (static_cast<uint32_t>(al->class_bit[c] + 8 * w * k) << 8);
    for (int i = 0; i < 4 && 4 * k + i < nb; ++i)
      al->plan_col_block[4 * x + i] = static_cast<int8_t>(al->stream_block[first + 4 * k + i]);
  }
  if (tid == 0) {
    al->plan_n_slots = n_slots;
    al->plan_k_cols = (4 * n_slots + 7) / 8 * 8;
  }
  // Digest of the allocation: sum mod 2^64 over blocks of splitmix64(b << 40 | w_b << 32 | g_b bits).
  if (tid < kH) {
    uint64_t z = (static_cast<uint64_t>(tid) << 40) | (static_cast<uint64_t>(sWidth[tid]) << 32) |
                 static_cast<uint64_t>(__float_as_uint(al->gain[tid]));
    z = splitmix64(z);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if ((tid & 31) == 0) sDig[tid >> 5] = z;
  }
  __syncthreads();
  if (tid == 0) al->digest = sDig[0] + sDig[1];
  __syncthreads();
  uint4* dst = reinterpret_cast<uint4*>(alloc + h);
  const uint4* src = reinterpret_cast<const uint4*>(&sRec);
  for (int i = tid; i < kRecWords / 4; i += blockDim.x) dst[i] = src[i];
}

}  // namespace kvq
