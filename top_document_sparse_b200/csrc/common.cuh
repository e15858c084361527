// common.cuh -- types and device helpers shared by the MSA kernels (one
// translation unit: msa.cu includes every kernel header).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "../../include/msa.h"

// The memory description behind the opaque msa_memory handle.
struct msa_memory {
  int32_t n_docs = 0, chunk_len = 0, H_kv = 0, D = 0, H_r = 0, d_r = 0;
  msa_dtype dtype = MSA_F32;
  double theta = 0.0;
  int32_t max_local_position = 0;
  int64_t n_tokens = 0, n_chunks = 0;
  int32_t max_doc_chunks = 0;
  int64_t max_doc_tokens = 0;
  int32_t rope_len = 0;
  int device = 0;
  std::vector<int64_t> doc_tok_off, doc_chunk_off;
  int32_t *d_chunk_doc = nullptr;      // [C] chunk -> document
  int64_t *d_doc_tok_off = nullptr;    // [n_docs + 1]
  int64_t *d_doc_chunk_off = nullptr;  // [n_docs + 1]
  float2 *d_rope = nullptr;            // [rope_len][D/2] (cos, sin)
};

namespace msa {

constexpr float kEps = 1e-12f;
constexpr int kMaxChunkLen = 64;   // leaves of the pairwise pooling tree
constexpr int kMaxTopK = 64;

// Device error word (see MSA_DEVERR_* in msa.h).
__device__ unsigned int g_device_error = 0u;

__device__ __forceinline__ void raise_device_error(unsigned int bits) {
  atomicOr(&g_device_error, bits);
}

// ---------------------------------------------------------------- element I/O
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float x) { return x; }
  static __device__ __forceinline__ float from_f(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// Load / store 4 consecutive elements (16 B for fp32, 8 B for bf16).
__device__ __forceinline__ void load4(const float *p, float v[4]) {
  float4 x = *reinterpret_cast<const float4 *>(p);
  v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16 *p, float v[4]) {
  uint2 x = *reinterpret_cast<const uint2 *>(p);
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&x.x);
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&x.y);
  float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  v[0] = fa.x; v[1] = fa.y; v[2] = fb.x; v[3] = fb.y;
}
__device__ __forceinline__ void store4(float *p, const float v[4]) {
  *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store4(__nv_bfloat16 *p, const float v[4]) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
  __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
  uint2 x;
  x.x = *reinterpret_cast<uint32_t *>(&a);
  x.y = *reinterpret_cast<uint32_t *>(&b);
  *reinterpret_cast<uint2 *>(p) = x;
}

// ---------------------------------------------------------------- float max
// Atomic max on a plain fp32 word (finite values and -inf): non-negative
// floats order like signed ints, negative floats order reversed as unsigned.
__device__ __forceinline__ void atomic_max_float(float *addr, float v) {
  if (v >= 0.0f)
    atomicMax(reinterpret_cast<int *>(addr), __float_as_int(v));
  else
    atomicMin(reinterpret_cast<unsigned int *>(addr), __float_as_uint(v));
}

// Order-preserving 64-bit key for top-k: larger score first, then lower id.
__device__ __forceinline__ unsigned long long topk_key(float s, int32_t id) {
  unsigned int u = __float_as_uint(s);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<unsigned long long>(u) << 32) |
         static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<unsigned int>(id));
}
__device__ __forceinline__ float topk_key_score(unsigned long long key) {
  unsigned int u = static_cast<unsigned int>(key >> 32);
  u = (u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u;
  return __uint_as_float(u);
}
__device__ __forceinline__ int32_t topk_key_id(unsigned long long key) {
  return static_cast<int32_t>(0xFFFFFFFFu - static_cast<unsigned int>(key & 0xFFFFFFFFull));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace msa
