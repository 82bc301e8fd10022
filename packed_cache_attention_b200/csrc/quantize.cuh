// Quantize + pack: TQ-MSE-style scalar quantizer with Block-GTQ widths for K and a uniform
// width for V (page "RoPE-aware bit allocation for KV cache quantization", abstract: the
// allocator sits on TurboQuant-MSE, K and V get matched bit budgets, the cache is packed).
//
// For a token row x (128 values):
//   s2   = sum_j x_j^2 in fp32: eight partial sums over j = r (mod 8), j ascending, each
//          step fl32(s_r + fl32(x_j x_j)), combined ((s0+s1)+(s2+s3))+((s4+s5)+(s6+s7))
//   norm = fp16(fp32 sqrt(s2)) (round to nearest even)
//   a    = fp32(sqrt(128)) / fp32(norm), 0 if norm == 0
//   y_j  = fp32(fp32(x_j a) g_b)            (V: g = 1, the multiply is skipped as exact)
//   code = #{thresholds of width w_b strictly below y_j}
//
// Work split. Persistent warps; one warp owns a 32-token tile of one (sequence, KV head) at
// a time. Each warp keeps two shared-memory tile buffers, one for K rows and one for V rows,
// filled by cp.async (16-byte pieces, zero fill past the sequence end) one half-task ahead:
// the next tile's K rows load while this tile's V codes are computed, and the next V rows
// while the next K codes are computed. Rows sit at a pitch of 16-byte pieces plus one
// (68 words for 16-bit inputs), so a lane reading 16 bytes of its own row and a warp
// reading one word of one row are both free of bank conflicts.
//
// Code search. Width 1 is the sign. Wider codebooks use a lookup table on a uniform grid
// of cells of 2^-max(w-2, 1) over [-R_w, R_w): no cell holds two thresholds, so for y in cell k
//   code = (thresholds below the cell) + (y > the threshold inside the cell, if any),
// with y brought into the grid by a saturating multiply-add (widths 2..7) or a clamp (width
// 8); NaN lands in the lowest cell and compares false, so a NaN scale yields code 0 (tokens
// past the sequence end are written as code 0). The cell index is read off an fp32
// multiply-add rounded toward minus infinity into [2^23, 2^24). This is the same count as a
// search over the sorted thresholds, ties going to the lower code, for every fp32 y.
//
// K: lane t quantizes token t and appends its codes, in the allocation's stream order, to a
//   32-bit accumulator; the accumulator fills at the same code for every lane, so each full
//   word is one coalesced 128-byte warp store (word-planar tile layout). Codes are built in
//   groups of blocks at compile-time bit positions (4 blocks for widths up to 4, else 2) and
//   each group is merged into the stream with one funnel shift.
// V: lane l quantizes dims 2l, 2l+1, 64+2l, 65+2l for the 32 tokens of the tile, placing
//   token t's code at bit bits_v * t of the dim's stream (positions known at compile time).
#pragma once

#include <cmath>
#include <cstring>

#include "common.cuh"

namespace kvq {

// a * b + c for two pairs in one instruction, each rounded toward -infinity.
__device__ __forceinline__ float2 fma2_rm(float2 a, float2 b, float2 c) {
  uint64_t ua, ub, uc, ud;
  memcpy(&ua, &a, 8);
  memcpy(&ub, &b, 8);
  memcpy(&uc, &c, 8);
  asm("fma.rm.f32x2 %0, %1, %2, %3;" : "=l"(ud) : "l"(ua), "l"(ub), "l"(uc));
  float2 d;
  memcpy(&d, &ud, 8);
  return d;
}

// ---------------------------------------------------------------- code lookup table

// Code of y for width w: the number of thresholds below y. A table maps y to a grid cell that
// holds at most one threshold; entry {below, tau} of a cell is the number of thresholds below
// its left edge and the threshold inside it (+inf if none), so code = below + (y > tau).
// Widths 2..7: y in [-R, R), R = 2^(p-1), is mapped to u = y 2^-p + 0.5 in [0, 1) by one
// multiply-add rounded down and saturated to [0, 1] (NaN to 0), and u to cell floor(u 2^q) by
// a second one (the magic constant 1.5 * 2^23 puts the cell index in the low bits). Both round
// down and 2^-q is a multiple of the spacing of fp32 values near u, so the cell is exactly
// that of the real y; y >= R lands in the extra cell 2^q (all thresholds below). Cells are
// 2^(p-q) = 1/s_w wide with s_w = 2^max(w-2, 1). Width 8 (1024 cells would not fit) clamps y
// to [-K/s, K/s) first and takes the cell from one multiply-add.
constexpr int kLutP[9] = {0, 0, 1, 2, 3, 3, 3, 3, 0};               // R = 2^(p-1)
constexpr int kLutQ[9] = {0, 0, 2, 3, 5, 6, 7, 8, 0};               // 2^q cells (+1)
constexpr int kLutHalf8 = 288;                                      // width 8: half-range in cells
constexpr int kLutOffset[9] = {0, 0, 0, 5, 14, 47, 112, 241, 498};
constexpr int kLutEntries = 498 + 2 * kLutHalf8;                    // 1074

__host__ __device__ constexpr int lut_scale(int w) { return 1 << (w > 3 ? w - 2 : 1); }

// Host: builds the table from the fp32 thresholds (all widths concatenated, width w at
// 2^w - w - 1). Returns false if a cell would hold two thresholds or a threshold falls outside
// the grid.
inline bool quant_lut_image(const float* thresholds, uint32_t* out /* 2 * kLutEntries */) {
  for (int w = 2; w <= 8; ++w) {
    const float* t = thresholds + ((1 << w) - w - 1);
    const int n = (1 << w) - 1;
    int cells;
    double lo0, cw;
    if (w <= 7) {
      cells = (1 << kLutQ[w]) + 1;
      cw = std::ldexp(1.0, kLutP[w] - kLutQ[w]);
      lo0 = -std::ldexp(1.0, kLutP[w] - 1);
      if (static_cast<double>(t[0]) < lo0 || static_cast<double>(t[n - 1]) >= -lo0) return false;
    } else {
      cells = 2 * kLutHalf8;
      cw = 1.0 / lut_scale(8);
      lo0 = -kLutHalf8 * cw;
      if (static_cast<double>(t[0]) < lo0 || static_cast<double>(t[n - 1]) >= -lo0) return false;
    }
    for (int k = 0; k < cells; ++k) {
      const double lo = lo0 + k * cw;
      const double hi = (w <= 7 && k == cells - 1) ? INFINITY : lo + cw;
      uint32_t below = 0, inside = 0, tau = 0x7f800000u;
      for (int i = 0; i < n; ++i) {
        const double ti = t[i];
        if (ti < lo) ++below;
        else if (ti < hi) {
          ++inside;
          uint32_t b;
          std::memcpy(&b, &t[i], 4);
          tau = b;
        }
      }
      if (inside > 1) return false;
      out[2 * (kLutOffset[w] + k)] = below;
      out[2 * (kLutOffset[w] + k) + 1] = tau;
    }
  }
  return true;
}

__device__ __align__(16) uint32_t g_quant_lut[2 * kLutEntries];

// Entry of table address `addr` (a shared-memory byte address) compared with y.
__device__ __forceinline__ uint32_t lut_entry_code(float y, uint32_t addr) {
  uint32_t below, tau;
  asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(below), "=r"(tau) : "r"(addr));
  return below + (y > __uint_as_float(tau) ? 1u : 0u);
}

// Codes of y.x and y.y for width W (1..8) from the table in shared memory (lut_s: its
// shared-memory address). The entry of cell k sits at lut_s + 8 (offset + k), and
// k = bits(f) - 0x4B400000, so the entry address is one multiply-add of bits(f) with a folded
// constant (32-bit shared addresses wrap, so the constant's own wrap-around is harmless).
template <int W>
__device__ __forceinline__ uint2 lut_code2(float2 y, uint32_t lut_s) {
  if constexpr (W == 1) {
    return make_uint2(y.x > 0.0f ? 1u : 0u, y.y > 0.0f ? 1u : 0u);
  } else {
    constexpr uint32_t base = 8u * (static_cast<uint32_t>(kLutOffset[W]) - 0x4B400000u);
    float2 f;
    if constexpr (W <= 7) {
      constexpr float sp = 1.0f / static_cast<float>(1 << kLutP[W]);
      constexpr float sq = static_cast<float>(1 << kLutQ[W]);
      float2 u;
      asm("fma.rm.sat.f32 %0, %1, %2, 0f3F000000;" : "=f"(u.x) : "f"(y.x), "f"(sp));
      asm("fma.rm.sat.f32 %0, %1, %2, 0f3F000000;" : "=f"(u.y) : "f"(y.y), "f"(sp));
      f = fma2_rm(u, make_float2(sq, sq), make_float2(12582912.0f, 12582912.0f));
    } else {
      constexpr float s = static_cast<float>(lut_scale(8));
      constexpr float lo = -static_cast<float>(kLutHalf8) / s;
      constexpr float hi = (static_cast<float>(kLutHalf8) - 0.5f) / s;   // inside the last cell
      const float c = 12582912.0f + static_cast<float>(kLutHalf8);       // 1.5 * 2^23 + K + floor(yc s)
      f.x = __fmaf_rd(fminf(fmaxf(y.x, lo), hi), s, c);                  // NaN -> lo
      f.y = __fmaf_rd(fminf(fmaxf(y.y, lo), hi), s, c);
    }
    return make_uint2(lut_entry_code(y.x, static_cast<uint32_t>(__float_as_int(f.x)) * 8u + (lut_s + base)),
                      lut_entry_code(y.y, static_cast<uint32_t>(__float_as_int(f.y)) * 8u + (lut_s + base)));
  }
}

// Two fp32 products in one instruction, each rounded to nearest even.
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  uint64_t ua, ub, ud;
  memcpy(&ua, &a, 8);
  memcpy(&ub, &b, 8);
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(ud) : "l"(ua), "l"(ub));
  float2 d;
  memcpy(&d, &ud, 8);
  return d;
}

// ---------------------------------------------------------------- tile staging

template <int DT> struct QTile {
  static constexpr int kRowWords = (DT == KVQ_F32) ? kD : kD / 2;
  static constexpr int kPitch = kRowWords + 4;                 // words; 16-byte aligned rows
  static constexpr int kWords = kTile * kPitch;
  static constexpr int kPieces = kRowWords / 4;                // 16-byte pieces per row
  static constexpr int kPerLane = kTile * kPieces / 32;        // pieces a lane copies
  static constexpr int kWarps = (DT == KVQ_F32) ? 6 : 12;      // warps per CTA (one CTA per SM)
};

// Starts the copy of tile rows r_lo .. r_hi - 1 into `dst` (row r_lo at `src`, rows
// `row_stride` elements apart); the other rows are zero-filled without reading global memory.
template <int DT>
__device__ __forceinline__ void tile_load_async(uint32_t* dst, const void* src, int64_t row_stride, int r_lo, int r_hi,
                                                int lane) {
  using Q = QTile<DT>;
  constexpr int esz = (DT == KVQ_F32) ? 4 : 2;
  const uint8_t* s8 = static_cast<const uint8_t*>(src);
  const uint32_t d0 = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
#pragma unroll
  for (int i = 0; i < Q::kPerLane; ++i) {
    const int idx = i * 32 + lane;
    const int r = idx / Q::kPieces, c = idx % Q::kPieces;
    const bool ok = r >= r_lo && r < r_hi;
    const uint8_t* g = ok ? s8 + static_cast<int64_t>(r - r_lo) * row_stride * esz + 16 * c : s8;
    const uint32_t d = d0 + 4u * static_cast<uint32_t>(r * Q::kPitch + 4 * c);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(g), "r"(ok ? 16 : 0) : "memory");
  }
}

// Two consecutive values of a staged 16-bit or fp32 row as fp32.
template <int DT>
__device__ __forceinline__ float2 unpack_pair(uint32_t w) {
  if constexpr (DT == KVQ_BF16) return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  else return __half22float2(*reinterpret_cast<const __half2*>(&w));
}

// Two fp32 sums in one instruction, each rounded to nearest even.
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  uint64_t ua, ub, ud;
  memcpy(&ua, &a, 8);
  memcpy(&ub, &b, 8);
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(ud) : "l"(ua), "l"(ub));
  float2 d;
  memcpy(&d, &ud, 8);
  return d;
}

// a * b + c for two pairs in one instruction, each rounded once.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  uint64_t ua, ub, uc, ud;
  memcpy(&ua, &a, 8);
  memcpy(&ub, &b, 8);
  memcpy(&uc, &c, 8);
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(ud) : "l"(ua), "l"(ub), "l"(uc));
  float2 d;
  memcpy(&d, &ud, 8);
  return d;
}

// fp16 norm of the lane's own staged row and the scale a = sqrt(128)/norm (0 for a zero norm).
// The sum of squares is fixed to eight partial sums s_r over the coordinates j = r (mod 8),
// j ascending, combined as ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7)); acc[i] holds
// (s_2i, s_2i+1). For 16-bit inputs x * x is exact in fp32, so one fused multiply-add per
// step rounds exactly like the product followed by the sum.
template <int DT>
__device__ __forceinline__ void row_norm_scale(const uint32_t* row, __half& n16, float& a) {
  float2 acc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int c = 0; c < QTile<DT>::kPieces; ++c) {
    const uint4 v = *reinterpret_cast<const uint4*>(row + 4 * c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    if constexpr (DT == KVQ_F32) {
      // piece c holds coordinates 4c .. 4c + 3: pairs (s0, s1), (s2, s3) or (s4, s5), (s6, s7)
      const int base = 2 * (c & 1);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float2 x = make_float2(__uint_as_float(w[2 * i]), __uint_as_float(w[2 * i + 1]));
        acc[base + i] = add2(acc[base + i], mul2(x, x));
      }
    } else {
      // piece c holds coordinates 8c .. 8c + 7: word i is the pair (s_2i, s_2i+1)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 x = unpack_pair<DT>(w[i]);
        acc[i] = fma2(x, x, acc[i]);
      }
    }
  }
  const float lo = __fadd_rn(__fadd_rn(acc[0].x, acc[0].y), __fadd_rn(acc[1].x, acc[1].y));
  const float hi = __fadd_rn(__fadd_rn(acc[2].x, acc[2].y), __fadd_rn(acc[3].x, acc[3].y));
  const float s2 = __fadd_rn(lo, hi);
  n16 = __float2half_rn(__fsqrt_rn(s2));
  const float nf = __half2float(n16);
  const float sqd = 11.313708305358887f;       // fp32(sqrt(128))
  a = (nf == 0.0f) ? 0.0f : __fdiv_rn(sqd, nf);
}

// ---------------------------------------------------------------- K codes

// Per-warp table of the current head's blocks in stream order (plus 4 padding entries that
// a partial group may read): {byte selector that moves the block's half of its word into
// place | byte offset of that word in a staged row << 16, g}.
struct KEntry {
  uint32_t selofs;
  float g;
};
constexpr int kKEntries = kH + 4;

// Bit stream writer for one lane's K codes; `fill` and `word` advance identically in every
// lane, so every flushed word is a full-warp store of one word-planar row.
struct KStream {
  uint32_t cur = 0;
  int fill = 0;
  int word = 0;
  bool store = true;      // false: this lane's token is not written (it precedes an append)
  // Appends the low `nbits` (1..32) bits of `buf` (higher bits zero).
  __device__ __forceinline__ void append(uint32_t buf, int nbits, uint32_t* __restrict__ kout, int lane) {
    const uint64_t sh = static_cast<uint64_t>(buf) << fill;
    cur |= static_cast<uint32_t>(sh);
    const int nf = fill + nbits;
    if (nf >= 32) {
      if (store) kout[word * kTile + lane] = cur;
      ++word;
      cur = static_cast<uint32_t>(sh >> 32);
      fill = nf - 32;
    } else {
      fill = nf;
    }
  }
};

// Values of dims b and b + 64 of block `e` from the lane's staged row.
// (The byte permute reads only the low 16 bits of its selector.)
template <int DT>
__device__ __forceinline__ float2 block_pair(const uint8_t* row, const KEntry& e) {
  const uint8_t* p = row + (e.selofs >> 16);
  if constexpr (DT == KVQ_F32) {
    return make_float2(*reinterpret_cast<const float*>(p), *reinterpret_cast<const float*>(p + 256));
  } else if constexpr (DT == KVQ_BF16) {
    const uint32_t w1 = *reinterpret_cast<const uint32_t*>(p);
    const uint32_t w2 = *reinterpret_cast<const uint32_t*>(p + 128);
    return make_float2(__uint_as_float(__byte_perm(w1, 0u, e.selofs)), __uint_as_float(__byte_perm(w2, 0u, e.selofs)));
  } else {
    const uint32_t w1 = *reinterpret_cast<const uint32_t*>(p);
    const uint32_t w2 = *reinterpret_cast<const uint32_t*>(p + 128);
    const uint32_t h2 = __byte_perm(w1, w2, e.selofs);
    return __half22float2(*reinterpret_cast<const __half2*>(&h2));
  }
}

// All blocks of one width class (entries first .. first + nb - 1).
template <int DT, int W>
__device__ __forceinline__ void quant_k_class(const uint8_t* row, float2 aa, const KEntry* __restrict__ ent, int nb,
                                              uint32_t lut, KStream& ks, uint32_t* __restrict__ kout,
                                              int lane) {
  constexpr int GB = (W <= 4) ? 4 : 2;                          // blocks per group: 2 W GB <= 32 bits
  for (int k = 0; k < nb; k += GB) {
    uint32_t buf = 0;
#pragma unroll
    for (int j = 0; j < GB; ++j) {
      const KEntry e = ent[k + j];
      const float2 x = block_pair<DT>(row, e);
      const float2 y = mul2(mul2(x, aa), make_float2(e.g, e.g));
      const uint2 c = lut_code2<W>(y, lut);
      buf += c.x << (2 * W * j);                            // disjoint bit fields: + is |
      buf += c.y << (2 * W * j + W);
    }
    const int left = nb - k;
    int nbits = 2 * W * GB;
    if (left < GB) {
      nbits = 2 * W * left;
      buf &= (1u << nbits) - 1u;
    }
    ks.append(buf, nbits, kout, lane);
  }
}

// ---------------------------------------------------------------- V codes

// Width BV for every dim. Lane l handles dims {2l, 2l+1} and {64+2l, 65+2l}; sA2[t] = {a, a}
// of token t (NaN for tokens not written). Word i of dim j goes to vout[128 i + j]. The first
// `keep_bits` bits of every dim stream (tokens that precede an append) keep their stored value.
template <int DT, int BV>
__device__ __forceinline__ void quant_v_tile(const uint32_t* rows, const float2* sA2, uint32_t lut,
                                             uint32_t* __restrict__ vout, int keep_bits, int lane) {
  using Q = QTile<DT>;
#pragma unroll 1
  for (int half = 0; half < 2; ++half) {
    const int j0 = 2 * lane + kH * half;
    uint32_t w0[BV], w1[BV];
#pragma unroll
    for (int i = 0; i < BV; ++i) { w0[i] = 0u; w1[i] = 0u; }
#pragma unroll
    for (int tok = 0; tok < kTile; ++tok) {
      float2 x;
      if constexpr (DT == KVQ_F32) x = *reinterpret_cast<const float2*>(rows + tok * Q::kPitch + j0);
      else x = unpack_pair<DT>(rows[tok * Q::kPitch + (j0 >> 1)]);
      const float2 y = mul2(x, sA2[tok]);
      const uint2 cc = lut_code2<BV>(y, lut);
      const uint32_t c0 = cc.x, c1 = cc.y;
      const int bit = BV * tok, wi = bit >> 5, sh = bit & 31;
      w0[wi] += c0 << sh;                                   // disjoint bit fields: + is |
      w1[wi] += c1 << sh;
      if (sh + BV > 32) {
        w0[wi + 1] += c0 >> (32 - sh);
        w1[wi + 1] += c1 >> (32 - sh);
      }
    }
    if (keep_bits > 0) {
#pragma unroll
      for (int i = 0; i < BV; ++i) {
        const int kb = keep_bits - 32 * i;
        if (kb > 0) {
          const uint32_t m = kb >= 32 ? ~0u : (1u << kb) - 1u;
          const uint2 old = *reinterpret_cast<const uint2*>(vout + i * kD + j0);
          w0[i] |= old.x & m;
          w1[i] |= old.y & m;
        }
      }
    }
#pragma unroll
    for (int i = 0; i < BV; ++i)
      *reinterpret_cast<uint2*>(vout + i * kD + j0) = make_uint2(w0[i], w1[i]);
  }
}

// ---------------------------------------------------------------- kernel

// Per-warp shared memory: K tile, V tile, 32 {a, a} pairs, the K entry table, 8 classes.
template <int DT> struct QWarpSmem {
  static constexpr int kBytes = 2 * 4 * QTile<DT>::kWords + kTile * 8 + kKEntries * 8 + 8 * 4;
};

// Packed-header handling of a quantize or append call.
struct QHeader {
  int mode;              // 0: leave it, 1: write it (a call starting at token 0), 2: check it
  int batch, capacity, hdr_bytes;
};

// Header fields and digests written by CTA 0 (one warp) of a call that starts at token 0.
__device__ __forceinline__ void write_packed_header(uint8_t* packed, const QHeader& qh, int n_kv_heads, int bits_k,
                                                    int bits_v, int rec_bytes, const kvq_head_alloc* alloc,
                                                    int lane) {
  uint32_t* w = reinterpret_cast<uint32_t*>(packed);
  for (int i = lane; i < qh.hdr_bytes / 4; i += 32) {
    uint32_t v = 0u;
    if (i == 0) v = 0x3151564Bu;                                             // "KVQ1"
    else if (i == 1) v = 1u | (static_cast<uint32_t>(kD) << 16);           // layout 1, head_dim
    else if (i == 2) v = static_cast<uint32_t>(bits_k) | (static_cast<uint32_t>(bits_v) << 8) |
                         (static_cast<uint32_t>(alloc->w_max & 0xff) << 16) |
                         (static_cast<uint32_t>(alloc->mode & 0xff) << 24);
    else if (i == 4) v = static_cast<uint32_t>(qh.batch);
    else if (i == 5) v = static_cast<uint32_t>(n_kv_heads);
    else if (i == 6) v = static_cast<uint32_t>(qh.capacity);
    else if (i == 7) v = static_cast<uint32_t>(rec_bytes);
    else if (i >= 16 && i < 16 + 2 * n_kv_heads) {
      const uint64_t d = alloc[(i - 16) >> 1].digest;
      v = static_cast<uint32_t>((i & 1) ? (d >> 32) : d);
    }
    w[i] = v;
  }
}

// An append (call not starting at token 0) may only extend a cache whose header names this
// layout, these shapes and widths, and the same allocation, and carries no status; otherwise
// it records KVQ_ERR_MISMATCH there (keeping an earlier status) and writes nothing.
__device__ __forceinline__ bool packed_header_ok(uint8_t* packed, const QHeader& qh, int n_kv_heads, int bits_k,
                                                 int bits_v, int rec_bytes, const kvq_head_alloc* alloc) {
  const kvq_packed_header* H = reinterpret_cast<const kvq_packed_header*>(packed);
  bool ok = H->status == 0 && H->magic == 0x3151564Bu && H->layout_version == 1 && H->head_dim == kD &&
            H->bits_k == bits_k && H->bits_v == bits_v && H->batch == qh.batch && H->n_kv_heads == n_kv_heads &&
            H->capacity == qh.capacity && static_cast<int>(H->record_bytes) == rec_bytes;
  const uint64_t* dig = reinterpret_cast<const uint64_t*>(packed + sizeof(kvq_packed_header));
  for (int h = 0; ok && h < n_kv_heads; ++h) ok = dig[h] == alloc[h].digest;
  if (!ok) atomicCAS(const_cast<uint32_t*>(&H->status), 0u, static_cast<uint32_t>(KVQ_ERR_MISMATCH));
  return ok;
}

// One instantiation per value width BVT (= bits_v; 0 = keys only), so registers are
// allocated for one value pass only.
template <int DT, int BVT>
__global__ void __launch_bounds__(QTile<DT>::kWarps * 32, 1) kvq_quant_pack(
    const typename Elem<DT>::T* __restrict__ K, int64_t ksb, int64_t ksh, int64_t kst,
    const typename Elem<DT>::T* __restrict__ V, int64_t vsb, int64_t vsh, int64_t vst,
    int t_begin, int t_end, int tile_lo, int n_tiles, int n_kv_heads, int tiles_cap,
    const kvq_head_alloc* __restrict__ alloc, int bits_k, int bits_v, uint8_t* __restrict__ packed, int rec_bytes,
    int n_tasks, QHeader qh) {
  using Q = QTile<DT>;
  constexpr int kWarps = Q::kWarps;
  constexpr bool kKeysOnly = BVT == 0;
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ int sHeaderOk;
  uint2* sLut = reinterpret_cast<uint2*>(smem);
  for (int i = threadIdx.x; i < kLutEntries; i += blockDim.x)
    sLut[i] = make_uint2(g_quant_lut[2 * i], g_quant_lut[2 * i + 1]);
  const uint32_t lut_s = static_cast<uint32_t>(__cvta_generic_to_shared(sLut));
  // The table is the library's own; the caller's memory is touched only after the previous
  // kernel in the stream is done with it (programmatic dependent launch).
  grid_dependency_wait();
  if (threadIdx.x == 0) sHeaderOk = (qh.mode == 2) ? packed_header_ok(packed, qh, n_kv_heads, bits_k, bits_v, rec_bytes, alloc) : 1;
  if (qh.mode == 1 && blockIdx.x == 0 && threadIdx.x < 32)
    write_packed_header(packed, qh, n_kv_heads, bits_k, bits_v, rec_bytes, alloc, threadIdx.x);
  __syncthreads();
  if (!sHeaderOk) return;
  uint8_t* records = packed + qh.hdr_bytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k_words = bits_k * kD;
  uint8_t* wbase = smem + kLutEntries * 8 + warp * QWarpSmem<DT>::kBytes;
  uint32_t* kbuf = reinterpret_cast<uint32_t*>(wbase);
  uint32_t* vbuf = kbuf + Q::kWords;                // keys only: the second K tile buffer
  float2* sA2 = reinterpret_cast<float2*>(vbuf + Q::kWords);
  KEntry* sEnt = reinterpret_cast<KEntry*>(sA2 + kTile);
  uint32_t* sCls = reinterpret_cast<uint32_t*>(sEnt + kKEntries);     // width | first << 8 | blocks << 16
  const uint32_t* myv = vbuf + lane * Q::kPitch;
  int cur_h = -1, n_cls = 0;

  const int stride = gridDim.x * kWarps;
  int task = blockIdx.x * kWarps + warp;

  // A task's tile, the tile rows it writes [r_lo, r_hi) and the input rows of r_lo. Input row
  // i holds token t_begin + i.
  auto task_src = [&](int tk, int& bh, int& tile, int& r_lo, int& r_hi, const typename Elem<DT>::T*& kp,
                      const typename Elem<DT>::T*& vp) {
    bh = tk / n_tiles;
    tile = tile_lo + (tk - bh * n_tiles);
    const int h = bh % n_kv_heads, b = bh / n_kv_heads;
    const int t0 = tile * kTile;
    r_lo = max(0, t_begin - t0);
    r_hi = min(kTile, t_end - t0);
    const int64_t i0 = static_cast<int64_t>(t0 + r_lo - t_begin);
    kp = K + b * ksb + h * ksh + i0 * kst;
    vp = kKeysOnly ? nullptr : V + b * vsb + h * vsh + i0 * vst;
  };

  // The current task's coordinates; each iteration computes the next task's.
  int bh = 0, tile = 0, r_lo = 0, r_hi = 0;
  bool write = false;
  int kb = 0;                                       // keys only: the K buffer of the current task
  if (task < n_tasks) {
    const typename Elem<DT>::T *kp, *vp;
    task_src(task, bh, tile, r_lo, r_hi, kp, vp);
    tile_load_async<DT>(kbuf, kp, kst, r_lo, r_hi, lane);
    cp_async_commit();
    if constexpr (!kKeysOnly) {
      tile_load_async<DT>(vbuf, vp, vst, r_lo, r_hi, lane);
      cp_async_commit();
    }
  }

  for (; task < n_tasks; task += stride) {
    const int h = bh % n_kv_heads;
    const bool mine = lane >= r_lo;               // token written by this call (or past its end)
    const bool valid = mine && lane < r_hi;       // token quantized by this call
    const int next = task + stride;
    int nbh = 0, ntile = 0, nlo = 0, nhi = 0;
    const typename Elem<DT>::T *nkp = nullptr, *nvp = nullptr;
    if (next < n_tasks) task_src(next, nbh, ntile, nlo, nhi, nkp, nvp);

    if (h != cur_h) {
      const kvq_head_alloc* al = alloc + h;
      write = al->k_words == k_words;             // allocation made for another budget: write nothing
      for (int i = lane; i < kKEntries; i += 32) {
        const int blk = (i < kH) ? al->stream_block[i] : 0xff;
        KEntry e{0x1044u, 0.0f};
        if (blk < kH) {
          const float g = al->gain[blk];
          if constexpr (DT == KVQ_F32) e = KEntry{(4u * blk) << 16, g};
          else if constexpr (DT == KVQ_BF16) e = KEntry{((4u * (blk >> 1)) << 16) | ((blk & 1) ? 0x3244u : 0x1044u), g};
          else e = KEntry{((4u * (blk >> 1)) << 16) | ((blk & 1) ? 0x7632u : 0x5410u), g};
        }
        sEnt[i] = e;
      }
      n_cls = min(max(al->n_classes, 0), 8);
      if (lane < 8)
        sCls[lane] = static_cast<uint32_t>(al->class_width[lane]) | (static_cast<uint32_t>(al->class_first[lane]) << 8) |
                     (static_cast<uint32_t>(al->class_blocks[lane]) << 16);
      __syncwarp();
      cur_h = h;
    }
    uint8_t* rec = records + (static_cast<size_t>(bh) * tiles_cap + tile) * rec_bytes;
    uint32_t* kout = reinterpret_cast<uint32_t*>(rec);
    uint16_t* norms = reinterpret_cast<uint16_t*>(kout + k_words);   // 32 K norms, then 32 V norms
    uint32_t* vout = kout + k_words + kTile;
    uint32_t* kcur = (kKeysOnly && kb) ? vbuf : kbuf;
    uint32_t* knext = (kKeysOnly && !kb) ? vbuf : kbuf;

    // ---------------------------------------------------------------- K (Block-GTQ widths)
    if constexpr (kKeysOnly) {
      // the next task's K rows load into the other buffer while this one is coded
      if (nkp) tile_load_async<DT>(knext, nkp, kst, nlo, nhi, lane);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<1>();                        // this task's K rows (its V rows may be in flight)
    }
    __syncwarp();
    if (write) {
      __half n16;
      float a;
      const uint32_t* myk = kcur + lane * Q::kPitch;
      row_norm_scale<DT>(myk, n16, a);
      if (mine) norms[lane] = valid ? __half_as_ushort(n16) : 0;
      if (!valid) a = __int_as_float(0x7fc00000);   // NaN: every code is 0
      const float2 aa = make_float2(a, a);
      const uint8_t* row = reinterpret_cast<const uint8_t*>(myk);
      KStream ks;
      ks.store = mine;
      for (int c = 0; c < n_cls; ++c) {
        const uint32_t e = sCls[c];
        const int w = e & 0xffu, first = (e >> 8) & 0xffu, nb = e >> 16;
        const KEntry* ent = sEnt + first;
        switch (w) {
          case 1: quant_k_class<DT, 1>(row, aa, ent, nb, lut_s, ks, kout, lane); break;
          case 2: quant_k_class<DT, 2>(row, aa, ent, nb, lut_s, ks, kout, lane); break;
          case 3: quant_k_class<DT, 3>(row, aa, ent, nb, lut_s, ks, kout, lane); break;
          case 4: quant_k_class<DT, 4>(row, aa, ent, nb, lut_s, ks, kout, lane); break;
          case 5: quant_k_class<DT, 5>(row, aa, ent, nb, lut_s, ks, kout, lane); break;
          case 6: quant_k_class<DT, 6>(row, aa, ent, nb, lut_s, ks, kout, lane); break;
          case 7: quant_k_class<DT, 7>(row, aa, ent, nb, lut_s, ks, kout, lane); break;
          default: quant_k_class<DT, 8>(row, aa, ent, nb, lut_s, ks, kout, lane); break;
        }
      }
    }
    __syncwarp();                               // every lane is done with the K tile
    if constexpr (kKeysOnly) {
      kb ^= 1;
    } else {
      if (nkp) tile_load_async<DT>(kbuf, nkp, kst, nlo, nhi, lane);
      cp_async_commit();

      // -------------------------------------------------------------- V (uniform width)
      cp_async_wait<1>();                        // this task's V rows (next K rows may be in flight)
      __syncwarp();
      if (write) {
        __half n16;
        float a;
        row_norm_scale<DT>(myv, n16, a);
        if (mine) norms[kTile + lane] = valid ? __half_as_ushort(n16) : 0;
        if (!valid) a = __int_as_float(0x7fc00000);
        sA2[lane] = make_float2(a, a);
        const int keep = bits_v * r_lo;
        __syncwarp();
        quant_v_tile<DT, BVT>(vbuf, sA2, lut_s, vout, keep, lane);
      }
      __syncwarp();                               // every lane is done with the V tile and sA2
      if (nvp) tile_load_async<DT>(vbuf, nvp, vst, nlo, nhi, lane);
      cp_async_commit();
    }
    bh = nbh; tile = ntile; r_lo = nlo; r_hi = nhi;
  }
  allow_dependents();                                       // this warp has no task left
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Dynamic shared memory of kvq_quant_pack: the code lookup table, then per warp the K and V
// tiles, the value scales, the K entry table and the class table.
inline size_t quant_smem_bytes(int dtype) {
  if (dtype == KVQ_F32) return kLutEntries * 8 + static_cast<size_t>(QTile<KVQ_F32>::kWarps) * QWarpSmem<KVQ_F32>::kBytes;
  return kLutEntries * 8 + static_cast<size_t>(QTile<KVQ_BF16>::kWarps) * QWarpSmem<KVQ_BF16>::kBytes;
}
inline int quant_warps(int dtype) { return dtype == KVQ_F32 ? QTile<KVQ_F32>::kWarps : QTile<KVQ_BF16>::kWarps; }

}  // namespace kvq
