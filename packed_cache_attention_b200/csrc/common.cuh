// Device-side helpers shared by the libkvq kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "kvq.h"
#include "tables.h"

namespace kvq {

constexpr int kTile = KVQ_TILE_TOKENS;   // tokens per packed tile
constexpr int kD = KVQ_HEAD_DIM;         // head dim of the kernels
constexpr int kH = kD / 2;               // RoPE blocks per head
constexpr int kCalibChunk = 64;          // tokens per fixed-order energy partial sum
constexpr float kLog2e = 1.4426950408889634f;

// Constant tables on the device (uploaded once per device from tables()).
struct DevTables {
  uint16_t centroid_f16[kCentroidCount];
  float threshold[kThresholdCount];
  float delta[9];
  float nf4[16];
  float nf4_mid[15];
};

// Device copy of the tables. This header is compiled into a single translation unit
// (kvq.cu), which owns the symbol and uploads it once per device.
__constant__ DevTables c_tab;

// Workspace status word: first 4 bytes of every workspace.
struct WsHeader {
  unsigned int status;
  unsigned int pad[31];   // keep the payload 128-byte aligned
};

// ---------------------------------------------------------------- element loads

template <int DT> struct Elem;
template <> struct Elem<KVQ_F32> {
  using T = float;
  __device__ __forceinline__ static float to_f32(float x) { return x; }
};
template <> struct Elem<KVQ_F16> {
  using T = __half;
  __device__ __forceinline__ static float to_f32(__half x) { return __half2float(x); }
};
template <> struct Elem<KVQ_BF16> {
  using T = __nv_bfloat16;
  __device__ __forceinline__ static float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
};

template <typename T>
__device__ __forceinline__ T bits_to(uint32_t b);
template <>
__device__ __forceinline__ __half bits_to<__half>(uint32_t b) { return __ushort_as_half(static_cast<unsigned short>(b)); }
template <>
__device__ __forceinline__ __nv_bfloat16 bits_to<__nv_bfloat16>(uint32_t b) {
  return __ushort_as_bfloat16(static_cast<unsigned short>(b));
}

// ---------------------------------------------------------------- bit helpers

__device__ __forceinline__ uint32_t pack_half2(__half lo, __half hi) {
  return static_cast<uint32_t>(__half_as_ushort(lo)) | (static_cast<uint32_t>(__half_as_ushort(hi)) << 16);
}

// The SplitMix64 output function (Steele, Lea and Flood, OOPSLA 2014): one 64-bit mix. Used
// for the allocation digest that ties a packed cache to the allocation it was written with.
__host__ __device__ __forceinline__ uint64_t splitmix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Ticket of a split merge: one atomic add at GPU scope with acquire-release order. Taken by one
// thread right after the CTA barrier that follows the CTA's writes of its partial result, it
// publishes those writes (release); for the thread that draws the last ticket it also makes
// the earlier arrivers' writes visible (acquire) to every thread past the next CTA barrier.
__device__ __forceinline__ unsigned ticket_add(unsigned* p, unsigned n = 1u) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(n) : "memory");
  return old;
}

// Programmatic dependent launch. A kernel launched with programmatic stream serialization may
// start while the previous kernel in its stream is still finishing; it must not touch memory
// that kernel may write (or read) before grid_dependency_wait(), which returns once the previous
// grid has completed and its writes are visible (at once for a normal launch).
// allow_dependents() lets the next such kernel start as soon as every CTA of this grid has
// called it or exited.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// Split an fp32 value into fp16 hi + lo with hi + lo == x to ~2^-22 relative.
__device__ __forceinline__ void split_hilo(float x, __half& hi, __half& lo) {
  hi = __float2half_rn(x);
  lo = __float2half_rn(x - __half2float(hi));
}

// ---------------------------------------------------------------- async copies (cp.async, 16 B)

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }
}  // namespace kvq
