// Fused decode attention read straight from the packed Block-GTQ cache (page "RoPE-aware bit
// allocation for KV cache quantization", abstract: attention served from the packed cache;
// the NQKV review's editorial extensions propose folding the table lookup into attention).
//
// Grid: (splits, batch * n_kv_heads), one CTA per SM. A CTA owns a contiguous range of
// 128-token chunks (4 tile records, contiguous in memory) of one (sequence, KV head).
// Four warpgroups each run their own chunk pipeline over chunks g, g + 4, g + 8, .. of the
// range, each with four compute warps (warps 4g .. 4g + 3, warp % 4 = tensor-memory quarter)
// and one issuer warp (warp 16 + g) whose first lane issues every copy and product:
//   load     whole chunks (one bulk copy of 4 records) into the warpgroup's ring of stages,
//            several chunks ahead;
//   keys     lane = token: 16 K-hat columns at a time (4 slots of the allocation's plan, each
//            4 block pairs of one width, looked up in shared-memory pair tables; batches of
//            widths <= 5 take one width-generic instruction sequence) go to a ring
//            of two 16-column tensor-memory buffers; the issuer runs S^T[128 tokens][16] +=
//            Khat x Q'^T (tcgen05.mma, M 128, N 16; Q' rows 0-7 fp16 high parts, 8-15 low
//            parts) on each buffer as soon as it is full, while the next one is filled;
//   values   lane = dim: V-hat^T rows (one fp16 pair of tokens per column) go to their own 64
//            columns while the S products run;
//   softmax  lane = token: logits s = S * key norm * 2^e (per row, log2 units); an online
//            softmax whose running maximum m is only raised when some logit of the chunk
//            exceeds it by more than 8: one OR vote over the warpgroup decides, and only then
//            are the chunk's row maxima exchanged and O rescaled in tensor memory;
//            P' = 2^(s - m - 8) * value norm / sqrt(d), split into fp16 hi + lo, is the B
//            operand of O;
//   O        the issuer runs O^T[128 dims][16] += Vhat^T x P'^T, accumulated over all of the
//            warpgroup's chunks in tensor memory.
// One issuing thread can have one product in flight at a time (about 130 cycles each at
// these shapes), so four issuers keep four independent chains going.
// Q' carries f_b, log2(e)/sqrt(d) and a per-row power of two that keeps its fp16 split in
// range; all threads build it once the tables land. The four warpgroups' (m, l, O) are
// combined in shared memory; up to 20 splits then meet at the last CTA to finish (acquire-
// release ticket), more in two levels: the last CTA of each group of about sqrt(splits) splits
// merges the group, and the last group to finish merges the groups and writes out = O / l.
// Launched with programmatic dependent launch: barrier setup, the tensor-memory allocation
// and the copy of the library's own tables run before the wait for the previous kernel in the
// stream; nothing of the caller's memory is read or written before it.
// Keys-only caches (the Block-GTQ page reports key errors with only the keys quantized): the values of each
// chunk arrive as dense bf16/fp16 rows next to the chunk's K records and are transposed into
// tensor memory (lane = dim); O then runs on bf16 (or fp16) operands with P' split to match.
// Recent tokens kept unquantized (our reading of the recent-token buffer the page names): the issuer
// warps of every CTA, once their products are issued, attend over an even share of them on
// CUDA cores (lane = 4 dims) and add a fifth partial to the CTA's combine.
// Every wait is bounded. A wait that gives up records KVQ_ERR_TIMEOUT and stops the
// warpgroup; the CTA waits (bounded) for its copies and products in flight, frees tensor
// memory and writes nothing. A packed header or allocation that does not match the call
// records KVQ_ERR_MISMATCH and writes nothing either.
#pragma once

#include "common.cuh"
#include "tcgen05.cuh"

namespace kvq {

constexpr int kDecWG = 4;                 // warpgroups
constexpr int kDecIssuerWarp0 = 4 * kDecWG;   // issuer warp of warpgroup g: 16 + g
constexpr int kDecThreads = 5 * kDecWG * 32;
constexpr int kChunkTiles = 4;
constexpr int kChunkTokens = kChunkTiles * kTile;   // = MMA M = tensor-memory lanes
constexpr int kStagesMax = 4;             // chunk stages per warpgroup
constexpr int kTau = 8;                   // lazy rescale threshold (log2 units)
constexpr uint32_t kTmemCols = 512;
constexpr int kPlanSlots = 24;
constexpr int kMergeMax = 64;             // group size bound of the split merge
constexpr int kMergeBatch = 10;           // merge entries loaded in one round trip
constexpr uint32_t kHeaderMagic = 0x3151564Bu;   // "KVQ1"
constexpr int kLayoutVersion = 1;

// Tensor-memory columns of warpgroup g: K-hat ring 2 x 16, V-hat^T 64, S 16, O 16.
__device__ __forceinline__ uint32_t col_k(int g, int slot) { return 128u * g + 16u * slot; }
__device__ __forceinline__ uint32_t col_v(int g) { return 128u * g + 32u; }
__device__ __forceinline__ uint32_t col_s(int g) { return 128u * g + 96u; }
__device__ __forceinline__ uint32_t col_o(int g) { return 128u * g + 112u; }

// Lookup-table image, built once per device (decode_lut_image) and bulk-copied into every
// CTA's shared memory at byte 0. Entries are fp16 centroid values c_w[e] of width w.
//   Pair tables, one 32-bit word per pair index i = code_a | code_b << w (the 2w bits of two
//   consecutive codes): {c[code_a], c[code_b]}. Widths 1..3 keep one copy per lane (entry i of
//   lane l at word 32 i + l), so the 32 lanes of a warp never share a bank; they sit at byte 0
//   (width 3, 8 KB), 8192 (width 2) and 10240 (width 1), so an entry's byte address is
//   base | i << 7 | lane << 2. Widths 4 and 5 keep one shared copy (1 KB and 4 KB).
//   Single tables of widths 6..8 (rare: the highest-energy blocks): one fp16 per code, shared.
__host__ __device__ constexpr int pair_off(int w) {
  return w == 3 ? 0 : w == 2 ? 8192 : w == 1 ? 10240 : w == 5 ? 10752 : 14848;
}
__host__ __device__ constexpr int single_off(int w) { return w == 6 ? 15872 : w == 7 ? 16000 : 16256; }
constexpr int kLutBytes = 16768;
// Shared-memory map (byte offsets from the start of dynamic shared memory).
constexpr int kAllocOff = kLutBytes;                 // copy of the KV head's kvq_head_alloc
constexpr int kBQOff = ((kAllocOff + static_cast<int>(sizeof(kvq_head_alloc)) + 127) / 128) * 128;
constexpr int kBQBytes = 8192;                       // Q' (B operand of S), K-major, <= 256 K elements
constexpr int kBPOff = kBQOff + kBQBytes;            // P' (B operand of O), one per warpgroup, N-major
constexpr int kBPBytes = 4096;
constexpr int kRecOff = kBPOff + kDecWG * kBPBytes;  // recent tokens' O share [8][128] fp32
constexpr int kRecQOff = kRecOff + 8 * kD * 4;       // recent tokens' q * log2(e) / sqrt(d) [8][128]
constexpr int kHdrOff = kRecQOff + 8 * kD * 4;
static_assert(kLutBytes % 16 == 0 && kAllocOff % 16 == 0 && sizeof(kvq_head_alloc) % 16 == 0,
              "bulk-copied regions must be 16-byte multiples");
static_assert(sizeof(kvq_head_alloc) == 2048 && sizeof(kvq_packed_header) == 64, "ABI record sizes");

struct DecHeader {
  uint64_t full[kDecWG][kStagesMax];   // chunk stage loaded
  uint64_t kready[kDecWG][2];          // K-hat ring buffer filled (4 compute warps)
  uint64_t kfree[kDecWG][2];           // K-hat ring buffer read by its S products
  uint64_t sfull[kDecWG];              // S of the chunk complete
  uint64_t vready[kDecWG];             // V-hat^T and P' written (4 compute warps)
  uint64_t ofull[kDecWG];              // O products of the chunk complete
  uint64_t drain[kDecWG];              // every product the issuer committed is complete
  uint64_t setup;                      // lookup tables + allocation record copied in
  uint32_t tmem_base;
  int bad;                             // header or allocation mismatch: the CTA writes nothing
  int wg_abort[kDecWG];                // a wait of this warpgroup gave up
  float qscale[8];                     // 2^e that undoes the range scaling of Q' row h
  float qmax[16];                      // Q' row maxima: [row][half of the dims]
  float xch[kDecWG][4][8];             // chunk maximum: [warpgroup][warp][row]
  float lred[kDecWG][4][8];            // row sums: [warpgroup][warp][row]
  float wg_m[kDecWG + 1][8];           // warpgroup (and recent-token) results: maximum
  float wg_l[kDecWG + 1][8];           //                                        and row sum
  float rx_m[4][8];                    // recent tokens: per issuer warp maximum
  float rx_l[4][8];                    //                                and row sum
  int last;                            // this CTA drew the last ticket of its merge group
  uint4 kdesc[kPlanSlots];             // per plan slot of width <= 5: word offset, shifts, mask, stride
  uint32_t kbase[kPlanSlots];          //                                 pair-table byte offset
  int bkind[kPlanSlots / 4];           // per batch of 4 slots: 0 all widths <= 5, 1 otherwise
};

__host__ __device__ constexpr int decode_stage_off() {
  return kHdrOff + ((static_cast<int>(sizeof(DecHeader)) + 127) / 128) * 128;
}

// Bytes of a chunk stage: 4 tile records.
__host__ __device__ constexpr int chunk_bytes(int rec_bytes) { return kChunkTiles * rec_bytes; }

// Host: the lookup-table image from the fp16 centroid table (width w at c16 + 2^w - 2).
inline void decode_lut_image(const uint16_t* c16, uint8_t* img) {
  for (int w = 1; w <= 5; ++w) {
    const uint16_t* c = c16 + (1 << w) - 2;
    uint32_t* t = reinterpret_cast<uint32_t*>(img + pair_off(w));
    const int copies = w <= 3 ? 32 : 1;
    for (int e = 0; e < (1 << (2 * w)); ++e)
      for (int l = 0; l < copies; ++l)
        t[e * copies + l] = static_cast<uint32_t>(c[e & ((1 << w) - 1)]) | (static_cast<uint32_t>(c[e >> w]) << 16);
  }
  for (int w = 6; w <= 8; ++w) {
    uint16_t* t = reinterpret_cast<uint16_t*>(img + single_off(w));
    for (int e = 0; e < (1 << w); ++e) t[e] = c16[(1 << w) - 2 + e];
  }
}

// Device copy of the image (single translation unit; uploaded once per device).
__device__ __align__(16) uint8_t g_dec_lut[kLutBytes];

// ---------------------------------------------------------------- code extraction + lookup

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
// of hi:lo; code_a goes to the low half. Widths 1..5: one pair-table lookup (per-lane copy for
// 1..3); widths 6..8: two single-code lookups.
template <int W>
__device__ __forceinline__ uint32_t pair_value(uint32_t lo, uint32_t hi, int p, const uint8_t* sm, uint32_t lane4) {
  if constexpr (W <= 3) {
    return *reinterpret_cast<const uint32_t*>(sm + pair_off(W) + (field_at(lo, hi, p, 2 * W, 7) | lane4));
  } else if constexpr (W <= 5) {
    return *reinterpret_cast<const uint32_t*>(sm + pair_off(W) + field_at(lo, hi, p, 2 * W, 2));
  } else {
    const uint8_t* t = sm + single_off(W);
    return static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(t + field_at(lo, hi, p, W, 1))) |
           (static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(t + field_at(lo, hi, p + W, W, 1))) << 16);
  }
}

// Lookups of one slot whose 2 aligned stream words r0:r1 (the slot's first code at bit 0) are
// already in registers: width W from the slot entry e (0: an empty slot, zeros).
__device__ __forceinline__ void k_slot_vals(uint32_t e, uint32_t r0, uint32_t r1, const uint8_t* sm, uint32_t lane4,
                                            uint32_t* v) {
  switch (e & 15u) {
#define KVQ_SLOT_CASE(W) \
  case W:                \
    _Pragma("unroll") for (int k = 0; k < 4; ++k) v[k] = pair_value<W>(r0, r1, 2 * W * k, sm, lane4); break;
    KVQ_SLOT_CASE(1)
    KVQ_SLOT_CASE(2)
    KVQ_SLOT_CASE(3)
    KVQ_SLOT_CASE(4)
    KVQ_SLOT_CASE(5)
    KVQ_SLOT_CASE(6)
    KVQ_SLOT_CASE(7)
    KVQ_SLOT_CASE(8)
#undef KVQ_SLOT_CASE
    default: v[0] = 0u; v[1] = 0u; v[2] = 0u; v[3] = 0u; break;
  }
}

// 16 K-hat columns (4 plan slots) of this lane's token. The stream words of all four slots
// are loaded and aligned before any width is dispatched, so the loads of one batch overlap
// and only the table lookups follow the per-slot switch. kw points at word 0 of the token
// (word i at kw[32 i]); every slot reads three words (the third lies inside the record).
__device__ __forceinline__ void k_batch(const uint32_t* kw, uint4 e4, const uint8_t* sm, uint32_t lane4,
                                        uint32_t (&v)[16]) {
  const uint32_t e[4] = {e4.x, e4.y, e4.z, e4.w};
  uint32_t r0[4], r1[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t off = e[i] >> 8, j0 = off >> 5, sh = off & 31u;
    const uint32_t x0 = kw[j0 * 32], x1 = kw[(j0 + 1) * 32], x2 = kw[(j0 + 2) * 32];
    r0[i] = __funnelshift_r(x0, x1, sh);
    r1[i] = __funnelshift_r(x1, x2, sh);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) k_slot_vals(e[i], r0[i], r1[i], sm, lane4, v + 4 * i);
}

// 16 K-hat columns (4 plan slots) of this lane's token when every slot's width is at most 5
// (or the slot is empty): the same instructions for every width, so the lookups of all four
// slots are issued back to back. A slot's descriptor holds the byte offset of the stream word
// with its first code (x), the bit shift of that code in the word and the shifts of its block
// pairs 1..3 (y: one per byte, each read modulo 32 by the funnel shifts), the pair-index mask
// (z) and the table stride (w: 128 for the per-lane tables of widths 1..3, 4 for the shared
// ones); base is the table's byte offset.
__device__ __forceinline__ void k_batch_gen(const uint32_t* kw, const uint4* desc, const uint32_t* base,
                                            const uint8_t* sm, uint32_t lane4, uint32_t (&v)[16]) {
  uint4 d[4];
  uint32_t r0[4], r1[4], lb[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    d[i] = desc[i];
    const uint32_t* p = reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint8_t*>(kw) + d[i].x);
    const uint32_t x0 = p[0], x1 = p[32], x2 = p[64];
    r0[i] = __funnelshift_r(x0, x1, d[i].y);
    r1[i] = __funnelshift_r(x1, x2, d[i].y);
    lb[i] = base[i] | (lane4 & (d[i].w - 4u));
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t t = (k == 0) ? r0[i] : __funnelshift_r(r0[i], r1[i], d[i].y >> (8 * k));
      v[4 * i + k] = *reinterpret_cast<const uint32_t*>(sm + (t & d[i].z) * d[i].w + lb[i]);
    }
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

// Named barrier over n threads that also returns the OR of `v` over them.
__device__ __forceinline__ bool named_sync_or(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(v ? 1u : 0u), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void record_status(unsigned* status, unsigned code) { atomicCAS(status, 0u, code); }

// Element i of a tensor of run-time dtype (kvq_dtype) as fp32.
__device__ __forceinline__ float load_f32(const void* p, int dtype, int64_t i) {
  if (dtype == KVQ_F32) return static_cast<const float*>(p)[i];
  if (dtype == KVQ_F16) return __half2float(static_cast<const __half*>(p)[i]);
  return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
}

// ---------------------------------------------------------------- kernel arguments

struct DecArgs {
  const void* q;
  int64_t qsb, qsh;
  int q_dtype;
  int n_q_heads, n_kv_heads, batch;
  // keys-only cache: dense values [batch][n_kv_heads][>= seq_len][128] (bf16 or fp16)
  const void* v_dense;
  int64_t vsb, vsh, vst;
  int cbytes;                        // bytes of a chunk stage (records, then dense value rows)
  // recent tokens kept unquantized: [batch][n_kv_heads][n_recent][128] keys and values
  const void* k_rec;
  const void* v_rec;
  int64_t krsb, krsh, krst, vrsb, vrsh, vrst;
  int kr_dtype, vr_dtype, n_recent;
  const uint8_t* packed;             // header at byte 0, records at byte hdr_bytes
  const kvq_head_alloc* alloc;
  int hdr_bytes, tiles_cap, rec_bytes, bits_k, bits_v, capacity;
  int seq_len, splits, n_groups, group_size, n_stages;
  float* out;
  float* part_m;                     // [bh][splits + n_groups][8]
  float* part_l;
  float* part_o;                     // [bh][splits + n_groups][8][128]
  unsigned* tickets;                 // [bh][ticket_stride]: final counter, then one per merge group
  int ticket_stride;
  unsigned* status;
  uint32_t wait_limit;
  int debug_no_loads;                // test hook: issue no copy, so every wait on a stage gives up
};

// ---------------------------------------------------------------- split merge

// Merges entries e0 .. e0 + n - 1 of row bh, each (m, l, O) with O unnormalized and m in log2
// units, into entry `dst_entry` (>= 0) or into out = O / l (dst_entry < 0). Thread (h, j4) of
// the first 256 keeps a running (M, L, O[4 j4 .. 4 j4 + 3]) of row h and folds the entries in
// kMergeBatch at a time: the loads of a batch are issued together, so a merge of up to
// kMergeBatch entries (every merge step when splits <= kMergeBatch^2) costs one round trip to
// L2 and no CTA barrier. The order of the sums is fixed.
__device__ __forceinline__ void merge_entries(const DecArgs& a, int bh, int pitch, int e0, int n, int dst_entry,
                                              float* out_bh, int G) {
  const int tid = threadIdx.x;
  if (tid >= 256) return;
  const int h = tid >> 5, j4 = tid & 31;
  const size_t row = static_cast<size_t>(bh) * pitch + e0;
  const float4* po = reinterpret_cast<const float4*>(a.part_o);
  float M = -INFINITY, L = 0.0f;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < n; s0 += kMergeBatch) {
    float mv[kMergeBatch], lv[kMergeBatch];
    float4 ov[kMergeBatch];
#pragma unroll
    for (int u = 0; u < kMergeBatch; ++u) {
      if (s0 + u < n) {
        const size_t e = row + s0 + u;
        mv[u] = __ldcg(a.part_m + e * 8 + h);
        lv[u] = __ldcg(a.part_l + e * 8 + h);
        ov[u] = __ldcg(po + (e * 8 + h) * (kD / 4) + j4);
      } else {
        mv[u] = -INFINITY;
        lv[u] = 0.0f;
        ov[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    float mx = M;
#pragma unroll
    for (int u = 0; u < kMergeBatch; ++u) mx = fmaxf(mx, mv[u]);
    if (mx == -INFINITY) continue;
    const float sc = (M == -INFINITY) ? 0.0f : fast_exp2(M - mx);
    L *= sc;
    o.x *= sc; o.y *= sc; o.z *= sc; o.w *= sc;
#pragma unroll
    for (int u = 0; u < kMergeBatch; ++u) {
      const float wt = (mv[u] == -INFINITY) ? 0.0f : fast_exp2(mv[u] - mx);
      L += lv[u] * wt;
      o.x += ov[u].x * wt; o.y += ov[u].y * wt; o.z += ov[u].z * wt; o.w += ov[u].w * wt;
    }
    M = mx;
  }
  if (dst_entry >= 0) {
    const size_t e = static_cast<size_t>(bh) * pitch + dst_entry;
    reinterpret_cast<float4*>(a.part_o)[(e * 8 + h) * (kD / 4) + j4] = o;
    if (j4 == 0) {
      a.part_m[e * 8 + h] = M;
      a.part_l[e * 8 + h] = L;
    }
  } else if (h < G) {
    const float inv = 1.0f / L;
    reinterpret_cast<float4*>(out_bh + static_cast<size_t>(h) * kD)[j4] =
        make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
  }
}

// ---------------------------------------------------------------- the kernel

// Dense value modes of kvq_decode_gtq (keys-only caches): bf16 or fp16 value rows.
constexpr int kDenseBf16 = 16;
constexpr int kDenseF16 = 17;

// Splits x into hi + lo of the 16-bit type of the O operands (bf16 when kBf, else fp16),
// returned as their bit patterns.
template <bool kBf>
__device__ __forceinline__ void split16(float x, uint32_t& hi, uint32_t& lo) {
  if constexpr (kBf) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    hi = __bfloat16_as_ushort(h);
    lo = __bfloat16_as_ushort(__float2bfloat16_rn(x - __bfloat162float(h)));
  } else {
    const __half h = __float2half_rn(x);
    hi = __half_as_ushort(h);
    lo = __half_as_ushort(__float2half_rn(x - __half2float(h)));
  }
}

// One instantiation per value mode VM: 1..8 = packed values of that width; kDenseBf16 /
// kDenseF16 = keys-only cache with dense value rows of that type.
template <int VM>
__global__ void __launch_bounds__(kDecThreads, 1) kvq_decode_gtq(const DecArgs a) {
  constexpr bool kDense = VM >= kDenseBf16;
  constexpr bool kBfO = VM == kDenseBf16;                  // O operands in bf16
  extern __shared__ __align__(1024) uint8_t sm[];
  DecHeader& S = *reinterpret_cast<DecHeader*>(sm + kHdrOff);
  uint8_t* stages = sm + decode_stage_off();
  float* rec_o = reinterpret_cast<float*>(sm + kRecOff);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.n_kv_heads, hkv = bh % a.n_kv_heads;
  const int G = a.n_q_heads / a.n_kv_heads;
  const kvq_head_alloc* al = a.alloc + hkv;
  const int n_tiles = (a.seq_len + kTile - 1) / kTile;
  const int n_chunks_all = (n_tiles + kChunkTiles - 1) / kChunkTiles;
  const int c_begin = static_cast<int>((static_cast<long long>(split) * n_chunks_all) / a.splits);
  const int c_end = static_cast<int>((static_cast<long long>(split + 1) * n_chunks_all) / a.splits);
  const int n_chunks = c_end - c_begin;
  const uint8_t* src = a.packed + a.hdr_bytes + static_cast<size_t>(bh) * a.tiles_cap * a.rec_bytes;
  const int cbytes = a.cbytes;
  const int kbytes = 4 * kD * a.bits_k;             // K words of a record
  const int NS = a.n_stages;
  const float inv_sqrt_d = 0.08838834764831845f;
  const uint32_t WL = a.wait_limit;

  // roles: compute warps 0..15 (warpgroup g = warp / 4, quarter q = warp % 4), issuer warps 16..19
  const bool is_issuer = warp >= kDecIssuerWarp0;
  const int g = is_issuer ? warp - kDecIssuerWarp0 : warp >> 2;
  const int q = warp & 3;
  const bool issuer = is_issuer && lane == 0;
  const int nj = (n_chunks > g) ? (n_chunks - g + kDecWG - 1) / kDecWG : 0;   // this warpgroup's chunks
  uint8_t* my_stages = stages + static_cast<size_t>(g) * NS * cbytes;

  // ------------------------------------------------------------------ barriers, TMEM, setup copy
  // Barrier initialisation, the tensor-memory allocation and the copy of the library's own
  // lookup tables read none of the caller's memory: they run before the wait for the previous
  // kernel in the stream (programmatic dependent launch), everything else after it.
  if (tid == 0) {
    for (int gg = 0; gg < kDecWG; ++gg) {
      for (int i = 0; i < kStagesMax; ++i) tc::mbar_init(&S.full[gg][i], 1);
      for (int i = 0; i < 2; ++i) {
        tc::mbar_init(&S.kready[gg][i], 4);
        tc::mbar_init(&S.kfree[gg][i], 1);
      }
      tc::mbar_init(&S.sfull[gg], 1);
      tc::mbar_init(&S.vready[gg], 4);
      tc::mbar_init(&S.ofull[gg], 1);
      tc::mbar_init(&S.drain[gg], 1);
      S.wg_abort[gg] = 0;
    }
    tc::mbar_init(&S.setup, 1);
    S.bad = 0;
    tc::mbar_fence_init();
    tc::mbar_arrive_expect_tx(&S.setup, kLutBytes + static_cast<uint32_t>(sizeof(kvq_head_alloc)));
    tc::bulk_g2s(sm, g_dec_lut, kLutBytes, &S.setup);
  }
  if (tid < 8) S.wg_m[kDecWG][tid] = -INFINITY;             // no recent share unless the issuers add one
  if (warp == kDecIssuerWarp0) tc::tmem_alloc(&S.tmem_base, kTmemCols);
  grid_dependency_wait();
  if (tid == 0) tc::bulk_g2s(sm + kAllocOff, al, sizeof(kvq_head_alloc), &S.setup);
  // Q' inputs: threads 0..511 each own two consecutive dims of one query row (row tid / 64);
  // their loads go out first, so their latency overlaps the setup below.
  const int qh = tid >> 6, qd = 2 * (tid & 63);
  float2 qin = make_float2(0.0f, 0.0f);
  if (tid < 512 && qh < G) {
    const int64_t qi = b * a.qsb + (hkv * G + qh) * a.qsh + qd;
    qin = make_float2(load_f32(a.q, a.q_dtype, qi), load_f32(a.q, a.q_dtype, qi + 1));
  }
  if (tid == 32) {
    // The packed header must name this layout, these widths and shapes, and this head's
    // allocation; a status left by an append is reported as is. All fields are loaded
    // before any is compared, so the loads overlap.
    const uint4 h0 = *reinterpret_cast<const uint4*>(a.packed);
    const uint4 h1 = *reinterpret_cast<const uint4*>(a.packed + 16);
    const uint64_t dg = reinterpret_cast<const uint64_t*>(a.packed + sizeof(kvq_packed_header))[hkv];
    const uint64_t ad = al->digest;
    const int abk = al->bits_k, akw = al->k_words, apk = al->plan_k_cols, aps = al->plan_n_slots;
    const uint32_t want2 = static_cast<uint32_t>(a.bits_k) | (static_cast<uint32_t>(a.bits_v) << 8);
    unsigned code = 0;
    if (h0.w != 0) {
      code = h0.w;                                          // status left by an append
    } else {
      const bool ok = (h0.x == kHeaderMagic) & (h0.y == (static_cast<uint32_t>(kLayoutVersion) | (kD << 16))) &
                      ((h0.z & 0xffffu) == want2) & (static_cast<int>(h1.x) == a.batch) &
                      (static_cast<int>(h1.y) == a.n_kv_heads) & (static_cast<int>(h1.z) == a.capacity) &
                      (static_cast<int>(h1.w) == a.rec_bytes) & (dg == ad) & (abk == a.bits_k) &
                      (akw == a.bits_k * kD) & (apk <= 96) & (apk >= 8) & (aps <= kPlanSlots);
      if (!ok) code = KVQ_ERR_MISMATCH;
    }
    if (code) {
      S.bad = 1;
      record_status(a.status, code);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = S.tmem_base;

  int issued = 0;                                           // chunks whose copy this issuer started
  auto issue_chunk = [&](int j) {                           // issuer only
    const int ci = c_begin + g + kDecWG * j;
    const int tile0 = ci * kChunkTiles;
    const int nt = min(kChunkTiles, n_tiles - tile0);
    const int s = j % NS;
    uint8_t* dst = my_stages + static_cast<size_t>(s) * cbytes;
    uint32_t bytes = static_cast<uint32_t>(nt * a.rec_bytes);
    int rows = 0;
    if constexpr (kDense) {
      rows = min(kChunkTokens, a.seq_len - ci * kChunkTokens);
      bytes += static_cast<uint32_t>(rows) * (2 * kD);
    }
    tc::mbar_arrive_expect_tx(&S.full[g][s], bytes);
    tc::bulk_g2s(dst, src + static_cast<size_t>(tile0) * a.rec_bytes, static_cast<uint32_t>(nt * a.rec_bytes),
                 &S.full[g][s]);
    if constexpr (kDense) {
      const uint8_t* vsrc = static_cast<const uint8_t*>(a.v_dense) +
                            2 * (b * a.vsb + hkv * a.vsh + static_cast<int64_t>(ci) * kChunkTokens * a.vst);
      uint8_t* vdst = dst + kChunkTiles * a.rec_bytes;
      if (a.vst == kD) {
        tc::bulk_g2s(vdst, vsrc, static_cast<uint32_t>(rows) * (2 * kD), &S.full[g][s]);
      } else {
        for (int r = 0; r < rows; ++r)
          tc::bulk_g2s(vdst + r * (2 * kD), vsrc + 2 * static_cast<int64_t>(r) * a.vst, 2 * kD, &S.full[g][s]);
      }
    }
  };
  // First copies go out before anything else, so HBM is busy from the start.
  if (issuer && !S.bad && !a.debug_no_loads) {
    for (; issued < min(NS, nj); ++issued) issue_chunk(issued);
  }
  if (!tc::mbar_wait(&S.setup, 0, WL)) {
    S.bad = 1;
    record_status(a.status, KVQ_ERR_TIMEOUT);
  }
  __syncthreads();
  const kvq_head_alloc& A = *reinterpret_cast<const kvq_head_alloc*>(sm + kAllocOff);
  // ------------------------------------------------------------------ slot descriptors, Q'
  // Q' row h: q_h * f_b * log2(e) / sqrt(d), scaled by 2^-e so its largest |value| is in
  // [0.5, 1); qscale[h] = 2^e multiplies the product back. Built by all threads in three steps
  // (row maxima, scaled rows, the B operand of S), one CTA barrier after each.
  float* qtmp = reinterpret_cast<float*>(sm + kRecQOff);    // [8][128] fp32
  if (tid < 512) {
    const float sc = inv_sqrt_d * kLog2e;
    qin.x *= A.dequant[qd % kH] * sc;
    qin.y *= A.dequant[(qd + 1) % kH] * sc;
    float mx = fmaxf(fabsf(qin.x), fabsf(qin.y));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) S.qmax[warp] = mx;
  } else if (tid < 512 + kPlanSlots) {
    // descriptor of plan slot i for the width-generic lookups (an empty slot reads the first
    // codes of the stream through the width-1 table: finite values against zero Q' rows); a
    // slot whose codes would start past the key stream marks the allocation unusable
    const int i = tid - 512;
    const uint32_t e = A.plan_slot[i];
    uint32_t w = e & 15u, off = e >> 8;
    if (w > 8 || (w > 0 && off >= static_cast<uint32_t>(kD * a.bits_k))) {
      S.bad = 1;
      record_status(a.status, KVQ_ERR_MISMATCH);
    }
    if (w == 0 || w > 5 || off >= static_cast<uint32_t>(kD * a.bits_k)) { w = 1; off = 0; }
    S.kdesc[i] = make_uint4((off >> 5) * 128u, (off & 31u) | (2 * w) << 8 | (4 * w) << 16 | (6 * w) << 24,
                            (1u << (2 * w)) - 1u, w <= 3 ? 128u : 4u);
    S.kbase[i] = static_cast<uint32_t>(pair_off(static_cast<int>(w)));
  } else if (tid >= 512 + 32 && tid < 512 + 32 + kPlanSlots / 4) {
    const int bt = tid - 512 - 32;
    uint32_t wmax = 0;
    for (int i = 0; i < 4; ++i) wmax = max(wmax, A.plan_slot[4 * bt + i] & 15u);
    S.bkind[bt] = wmax <= 5 ? 0 : 1;
  }
  __syncthreads();
  if (tid < 512) {
    const float mx = fmaxf(S.qmax[2 * qh], S.qmax[2 * qh + 1]);
    int e = 0;
    if (mx > 0.0f) frexpf(mx, &e);
    const float sc = ldexpf(1.0f, -e);
    *reinterpret_cast<float2*>(qtmp + qh * kD + qd) = make_float2(qin.x * sc, qin.y * sc);
    if ((tid & 63) == 0) S.qscale[qh] = ldexpf(1.0f, e);
  }
  __syncthreads();
  {
    // B operand of S, K-major, no swizzle: element (n, k) at (k/8)*256 + (n/8)*128 + (n%8)*16 +
    // (k%8)*2; K element k = 2c + r is dim b + 64 r of the block in column c; n < 8: hi part of
    // row n, n >= 8: lo part.
    const int k_elems = 2 * min(max(A.plan_k_cols, 0), 96);
    for (int i = tid; i < 8 * k_elems; i += blockDim.x) {
      const int n = i / k_elems, k = i - n * k_elems;
      const int blk = A.plan_col_block[k >> 1];
      __half hi = __float2half_rn(0.0f), lo = hi;
      if (blk >= 0 && blk < kH) split_hilo(qtmp[n * kD + blk + kH * (k & 1)], hi, lo);
      const int base = (k >> 3) * 256 + (k & 7) * 2;
      *reinterpret_cast<__half*>(sm + kBQOff + base + n * 16) = hi;
      *reinterpret_cast<__half*>(sm + kBQOff + base + 128 + n * 16) = lo;
    }
  }
  tc::fence_proxy_async_smem();
  __syncthreads();
  const bool bad = S.bad != 0;
  volatile int* abort_flag = &S.wg_abort[g];

  float M[8], L[8];                                         // running max (log2) and row sums
#pragma unroll
  for (int h = 0; h < 8; ++h) { M[h] = -INFINITY; L[h] = 0.0f; }
  int done = 0;                                             // chunks this warpgroup completed

  if (!bad && is_issuer) {
    const int it = tid - 32 * kDecIssuerWarp0;              // 0..127
    // ---------------------------------------------------------------- issuing (one lane per warpgroup)
    if (issuer) {
      const uint32_t id_s = tc::idesc_f16(128, 16, false), id_o = tc::idesc_f16(128, 16, true, kBfO);
      const uint32_t bq = tc::smem_u32(sm + kBQOff), bp = tc::smem_u32(sm + kBPOff + g * kBPBytes);
      const int nb = (min(A.plan_n_slots, kPlanSlots) + 3) >> 2;
      const int k_steps = A.plan_k_cols >> 3;
      const uint32_t tS = tbase + col_s(g), tO = tbase + col_o(g), tV = tbase + col_v(g);
      bool ok = true;
      for (int j = 0; j < nj && ok; ++j) {
        for (int bt = 0; bt < nb; ++bt) {
          const int kb = j * nb + bt, slot = kb & 1;
          if (!tc::mbar_wait(&S.kready[g][slot], (kb >> 1) & 1, WL)) { ok = false; break; }
          tc::fence_after_sync();
          const uint32_t tK = tbase + col_k(g, slot);
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int ks = 2 * bt + i;
            if (ks < k_steps) tc::mma_ts(tS, tK + 8 * i, tc::sdesc(bq + 512 * ks, 256, 128), id_s, ks > 0 ? 1u : 0u);
          }
          tc::mma_commit(&S.kfree[g][slot]);
        }
        if (!ok) break;
        tc::mma_commit(&S.sfull[g]);
        if (!tc::mbar_wait(&S.vready[g], j & 1, WL)) { ok = false; break; }
        tc::fence_after_sync();
#pragma unroll
        for (int ks = 0; ks < kChunkTokens / 16; ++ks)
          tc::mma_ts(tO, tV + 8 * ks, tc::sdesc(bp + 512 * ks, 256, 128), id_o, (j > 0 || ks > 0) ? 1u : 0u);
        tc::mma_commit(&S.ofull[g]);
        // the stage is consumed (keys, values and norms): refill it with a later chunk
        if (issued < nj && !a.debug_no_loads) issue_chunk(issued++);
      }
      if (!ok) *abort_flag = 1;
      // every product committed so far completes before the CTA can free tensor memory, and
      // every copy started lands before the CTA can leave
      tc::mma_commit(&S.drain[g]);
      tc::mbar_wait(&S.drain[g], 0, WL);
      for (int s = 0; s < NS; ++s) {
        int last = -1;
        for (int j = s; j < issued; j += NS) last = j;
        if (last >= 0) tc::mbar_wait(&S.full[g][s], (last / NS) & 1, WL);
      }
    }
    __syncwarp();
    // ---------------------------------------------------------------- recent tokens (CUDA cores)
    // This CTA's even share of the row's recent tokens. Lane l owns dims l, l + 32, l + 64,
    // l + 96; issuer warp w walks every fourth token with its own online softmax over
    // s = q . k * log2(e) / sqrt(d); the four warps then meet at a common maximum and add
    // their O shares into rec_o in a fixed order.
    const int r_begin = static_cast<int>((static_cast<long long>(split) * a.n_recent) / a.splits);
    const int r_end = static_cast<int>((static_cast<long long>(split + 1) * a.n_recent) / a.splits);
    if (r_end > r_begin) {
      const int w = g;
      float* rq = reinterpret_cast<float*>(sm + kRecQOff);  // reused: q * log2(e) / sqrt(d)
      named_sync(kDecWG + 1, 128);
      for (int i = it; i < 8 * kD; i += 128) {
        const int h = i >> 7, j = i & (kD - 1);
        rq[i] = (h < G) ? load_f32(a.q, a.q_dtype, b * a.qsb + (hkv * G + h) * a.qsh + j) * (inv_sqrt_d * kLog2e) : 0.0f;
      }
      named_sync(kDecWG + 1, 128);
      float o[8][4];
#pragma unroll
      for (int h = 0; h < 8; ++h)
#pragma unroll
        for (int u = 0; u < 4; ++u) o[h][u] = 0.0f;
      for (int r = r_begin + w; r < r_end; r += kDecWG) {
        float kv[4], vv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          kv[u] = load_f32(a.k_rec, a.kr_dtype, b * a.krsb + hkv * a.krsh + r * a.krst + lane + 32 * u);
          vv[u] = load_f32(a.v_rec, a.vr_dtype, b * a.vrsb + hkv * a.vrsh + r * a.vrst + lane + 32 * u);
        }
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          const float* qh = rq + h * kD + lane;
          float sdot = qh[0] * kv[0] + qh[32] * kv[1] + qh[64] * kv[2] + qh[96] * kv[3];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) sdot += __shfl_xor_sync(0xffffffffu, sdot, off);
          const float mn = fmaxf(M[h], sdot);
          const float alpha = (M[h] == -INFINITY) ? 0.0f : fast_exp2(M[h] - mn);
          const float p = fast_exp2(sdot - mn);
          M[h] = mn;
          L[h] = L[h] * alpha + p;
#pragma unroll
          for (int u = 0; u < 4; ++u) o[h][u] = o[h][u] * alpha + p * vv[u];
        }
      }
      if (lane == 0) {
#pragma unroll
        for (int h = 0; h < 8; ++h) { S.rx_m[w][h] = M[h]; S.rx_l[w][h] = L[h]; }
      }
      named_sync(kDecWG + 1, 128);
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        const float Mx = fmaxf(fmaxf(S.rx_m[0][h], S.rx_m[1][h]), fmaxf(S.rx_m[2][h], S.rx_m[3][h]));
        const float wt = (M[h] == -INFINITY) ? 0.0f : fast_exp2(M[h] - Mx);
#pragma unroll
        for (int u = 0; u < 4; ++u) o[h][u] *= wt;
        if (w == 0 && lane == 0) {
          float lsum = 0.0f;
#pragma unroll
          for (int ww = 0; ww < 4; ++ww)
            lsum += (S.rx_m[ww][h] == -INFINITY) ? 0.0f : S.rx_l[ww][h] * fast_exp2(S.rx_m[ww][h] - Mx);
          S.wg_m[kDecWG][h] = Mx;
          S.wg_l[kDecWG][h] = lsum;
        }
      }
      for (int ww = 0; ww < kDecWG; ++ww) {
        if (w == ww) {
#pragma unroll
          for (int h = 0; h < 8; ++h)
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              float* dst = rec_o + h * kD + lane + 32 * u;
              *dst = (ww == 0) ? o[h][u] : *dst + o[h][u];
            }
        }
        named_sync(kDecWG + 1, 128);
      }
#pragma unroll
      for (int h = 0; h < 8; ++h) { M[h] = -INFINITY; L[h] = 0.0f; }
    }
  } else if (!bad) {
    // ------------------------------------------------------------------ compute warps
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    const uint32_t lane4 = static_cast<uint32_t>(lane) << 2;
    const uint32_t tV = tbase + col_v(g), tS = tbase + col_s(g), tO = tbase + col_o(g);
    const int nb = (min(A.plan_n_slots, kPlanSlots) + 3) >> 2;
    uint8_t* pbuf = sm + kBPOff + g * kBPBytes;
    const uint4* slots4 = reinterpret_cast<const uint4*>(A.plan_slot);
    float qs[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) qs[h] = S.qscale[h];

    for (int j = 0; j < nj; ++j) {
      const int ci = c_begin + g + kDecWG * j;
      const int s = j % NS;
      const uint8_t* st = my_stages + static_cast<size_t>(s) * cbytes;
      if (!tc::mbar_wait(&S.full[g][s], (j / NS) & 1, WL)) *abort_flag = 1;
      // -------------------------------------------------------------- keys (lane = token)
      const uint8_t* tq = st + q * a.rec_bytes;                       // tile q of the chunk
      const uint32_t* kw = reinterpret_cast<const uint32_t*>(tq) + lane;
      // Batch bt's lookups run before the wait for batch bt - 1's store, so the store's
      // latency hides behind them; a ring buffer is refilled once its S products are done.
      for (int bt = 0; bt < nb; ++bt) {
        const int kb = j * nb + bt, slot = kb & 1;
        uint32_t v16[16];
        if (S.bkind[bt] == 0) k_batch_gen(kw, S.kdesc + 4 * bt, S.kbase + 4 * bt, sm, lane4, v16);
        else k_batch(kw, slots4[bt], sm, lane4, v16);
        if (bt > 0) {
          tc::wait_st();
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&S.kready[g][slot ^ 1]);
        }
        if (kb >= 2 && !tc::mbar_wait(&S.kfree[g][slot], ((kb >> 1) - 1) & 1, WL)) *abort_flag = 1;
        tc::fence_after_sync();
        tc::tmem_st<16>(tbase + col_k(g, slot) + lane_base, v16);
      }
      tc::wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&S.kready[g][(j * nb + nb - 1) & 1]);
      const float kn = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(tq + kbytes)[lane]));
      float vn = 1.0f;
      if constexpr (!kDense) vn = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(tq + kbytes + 2 * kTile)[lane]));
      const int tok0 = ci * kChunkTokens;
      const bool valid = tok0 + 32 * q + lane < a.seq_len;
      // -------------------------------------------------------------- values (lane = dim)
      // V-hat^T and P' are free once the previous chunk's O products are complete
      if (j > 0 && !tc::mbar_wait(&S.ofull[g], (j - 1) & 1, WL)) *abort_flag = 1;
      tc::fence_after_sync();
      if constexpr (kDense) {
        // dense rows [token][128] of 16-bit values after the chunk's records; rows past the
        // sequence end are not copied and read as 0
        const uint16_t* vr = reinterpret_cast<const uint16_t*>(st + kChunkTiles * a.rec_bytes) + 32 * q + lane;
        const int nrows = a.seq_len - tok0;
#pragma unroll
        for (int u = 0; u < kChunkTiles; ++u) {
          uint32_t v[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int t0 = 32 * u + 2 * c;
            const uint32_t lo = (t0 < nrows) ? vr[t0 * kD] : 0u;
            const uint32_t hi = (t0 + 1 < nrows) ? vr[(t0 + 1) * kD] : 0u;
            v[c] = lo | (hi << 16);
          }
          tc::tmem_st<16>(tV + lane_base + 16 * u, v);
        }
      } else {
#pragma unroll
        for (int u = 0; u < kChunkTiles; ++u) {
          const uint32_t* vw = reinterpret_cast<const uint32_t*>(st + u * a.rec_bytes + kbytes + 4 * kTile) + 32 * q + lane;
          v_tile<VM>(vw, tV + lane_base + 16 * u, sm, lane4);
        }
      }
      // -------------------------------------------------------------- logits
      if (!tc::mbar_wait(&S.sfull[g], j & 1, WL)) *abort_flag = 1;
      tc::fence_after_sync();
      float sv[8];
      {
        uint32_t sr[16];
        tc::tmem_ld<16>(tS + lane_base, sr);
        tc::wait_ld();
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          const float x = (__uint_as_float(sr[h]) + __uint_as_float(sr[8 + h])) * (kn * qs[h]);
          sv[h] = valid ? x : -INFINITY;
        }
      }
      // -------------------------------------------------------------- chunk maximum
      // The running maximum moves only when a logit of the chunk exceeds it by more than tau
      // (log2 units: a factor 2^tau once exponentiated). One barrier with an OR vote over the
      // warpgroup finds out; only then are the row maxima of the chunk exchanged and O
      // rescaled.
      bool over = false;
#pragma unroll
      for (int h = 0; h < 8; ++h) over |= sv[h] > M[h] + static_cast<float>(kTau);
      const bool any_over = named_sync_or(1 + g, 128, over);
      if (*abort_flag) break;
      if (any_over) {
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          const int m = __reduce_max_sync(0xffffffffu, ordered(sv[h]));
          if (lane == 0) S.xch[g][q][h] = from_ordered(m);
        }
        named_sync(1 + g, 128);
        float alpha[8];
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          const float cm = fmaxf(fmaxf(S.xch[g][0][h], S.xch[g][1][h]), fmaxf(S.xch[g][2][h], S.xch[g][3][h]));
          const float mn = fmaxf(M[h], cm);
          alpha[h] = (M[h] == -INFINITY) ? 0.0f : fast_exp2(M[h] - mn);
          M[h] = mn;
          L[h] *= alpha[h];
        }
        if (j > 0) {                                  // O holds earlier chunks: rescale it (lane = dim)
          uint32_t o[16];
          tc::tmem_ld<16>(tO + lane_base, o);
          tc::wait_ld();
#pragma unroll
          for (int c = 0; c < 16; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha[c & 7]);
          tc::tmem_st<16>(tO + lane_base, o);
        }
      }
      // -------------------------------------------------------------- P' (lane = token)
      {
        // packed values: P' = p * value norm / sqrt(d) (v-hat = norm * c / sqrt(d)); dense: p
        const float vs = valid ? (kDense ? 1.0f : vn * inv_sqrt_d) / static_cast<float>(1 << kTau) : 0.0f;
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int h = 0; h < 8; h += 2) {
          const float p0 = valid ? fast_exp2(sv[h] - M[h]) : 0.0f;
          const float p1 = valid ? fast_exp2(sv[h + 1] - M[h + 1]) : 0.0f;
          L[h] += p0;
          L[h + 1] += p1;
          uint32_t h0, l0, h1, l1;
          split16<kBfO>(p0 * vs, h0, l0);
          split16<kBfO>(p1 * vs, h1, l1);
          hi[h >> 1] = h0 | (h1 << 16);
          lo[h >> 1] = l0 | (l1 << 16);
        }
        const int t = 32 * q + lane;
        uint8_t* pb = pbuf + (t >> 3) * 256 + (t & 7) * 16;
        *reinterpret_cast<uint4*>(pb) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(pb + 128) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      tc::fence_proxy_async_smem();
      tc::wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&S.vready[g]);
      done = j + 1;
    }
    // ------------------------------------------------------------------ warpgroup result
    if (done > 0 && !*abort_flag && !tc::mbar_wait(&S.ofull[g], (done - 1) & 1, WL)) *abort_flag = 1;
    named_sync(1 + g, 128);
    tc::fence_after_sync();
    if (!*abort_flag) {
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        float l = L[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (lane == 0) S.lred[g][q][h] = l;
      }
    }
  } else if (issuer) {
    // a mismatched CTA still waits for the copies its issuer started
    for (int s = 0; s < NS; ++s) {
      int last = -1;
      for (int j = s; j < issued; j += NS) last = j;
      if (last >= 0) tc::mbar_wait(&S.full[g][s], (last / NS) & 1, WL);
    }
  }
  __syncthreads();
  allow_dependents();                                       // the next kernel may start on freed SMs
  bool aborted = bad;
#pragma unroll
  for (int gg = 0; gg < kDecWG; ++gg) aborted |= S.wg_abort[gg] != 0;
  if (aborted && !bad && tid == 0) record_status(a.status, KVQ_ERR_TIMEOUT);

  // ------------------------------------------------------------------ CTA result
  // Warpgroup partials (m, l, O) combined in shared memory (the stage area is free now).
  float* comb = reinterpret_cast<float*>(stages);           // [kDecWG][8][128] O, unscaled
  if (!aborted && !is_issuer) {
    const int d = 32 * q + lane;
    if (nj > 0) {
      uint32_t o[16];
      tc::tmem_ld<16>(tbase + col_o(g) + (static_cast<uint32_t>(32 * q) << 16), o);
      tc::wait_ld();
#pragma unroll
      for (int h = 0; h < 8; ++h)
        comb[(g * 8 + h) * kD + d] = (__uint_as_float(o[h]) + __uint_as_float(o[8 + h])) * static_cast<float>(1 << kTau);
    }
    const int tid_wg = 32 * q + lane;
    if (tid_wg < 8) {
      const int h = tid_wg;
      float mh = -INFINITY;
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r == h) mh = M[r];                        // (a register array is never indexed at run time)
      S.wg_m[g][h] = nj > 0 ? mh : -INFINITY;
      S.wg_l[g][h] = nj > 0 ? (S.lred[g][0][h] + S.lred[g][1][h] + S.lred[g][2][h] + S.lred[g][3][h]) : 0.0f;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == kDecIssuerWarp0) tc::tmem_dealloc(tbase, kTmemCols);
  if (aborted) return;

  const int pitch = a.splits + a.n_groups;
  float* out_bh = a.out + (static_cast<size_t>(b) * a.n_q_heads + hkv * G) * kD;
  // combine the warpgroups and the recent share: m = max, l and O = sums weighted by 2^(m_g - m)
  for (int i = tid; i < 8 * kD; i += blockDim.x) {
    const int h = i >> 7, d = i & (kD - 1);
    float Mx = -INFINITY;
#pragma unroll
    for (int gg = 0; gg <= kDecWG; ++gg) Mx = fmaxf(Mx, S.wg_m[gg][h]);
    float Ls = 0.0f, Os = 0.0f;
#pragma unroll
    for (int gg = 0; gg <= kDecWG; ++gg) {
      if (S.wg_m[gg][h] == -INFINITY) continue;
      const float w = fast_exp2(S.wg_m[gg][h] - Mx);
      Ls += w * S.wg_l[gg][h];
      Os += w * (gg < kDecWG ? comb[(gg * 8 + h) * kD + d] : rec_o[h * kD + d]);
    }
    if (a.splits == 1) {
      if (h < G) out_bh[h * kD + d] = Os / Ls;
    } else {
      const size_t e = static_cast<size_t>(bh) * pitch + split;
      a.part_o[(e * 8 + h) * kD + d] = Os;
      if (d == 0) {
        a.part_m[e * 8 + h] = Mx;
        a.part_l[e * 8 + h] = Ls;
      }
    }
  }
  if (a.splits == 1) return;

  // ------------------------------------------------------------------ split merge (one or two levels)
  // The last CTA of each group of splits (ticket order) merges the group; the last group to
  // finish merges the groups. A ticket is taken after the barrier that follows the writes it
  // publishes, with acquire-release order at GPU scope (no separate fences).
  const int grp = split / a.group_size;
  const int m0 = grp * a.group_size, m1 = min(a.splits, m0 + a.group_size);
  unsigned* tk = a.tickets + static_cast<size_t>(bh) * a.ticket_stride;
  __syncthreads();
  if (tid == 0) {
    const unsigned t = ticket_add(&tk[1 + grp]);
    S.last = (t == static_cast<unsigned>(m1 - m0 - 1));
    if (S.last) tk[1 + grp] = 0u;
  }
  __syncthreads();
  if (!S.last) return;
  if (a.n_groups == 1) {
    merge_entries(a, bh, pitch, m0, m1 - m0, -1, out_bh, G);
    return;
  }
  merge_entries(a, bh, pitch, m0, m1 - m0, a.splits + grp, out_bh, G);
  __syncthreads();
  if (tid == 0) {
    const unsigned t = ticket_add(&tk[0]);
    S.last = (t == static_cast<unsigned>(a.n_groups - 1));
    if (S.last) tk[0] = 0u;
  }
  __syncthreads();
  if (!S.last) return;
  merge_entries(a, bh, pitch, a.splits, a.n_groups, -1, out_bh, G);
}

}  // namespace kvq
