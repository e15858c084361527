// pool.cuh -- offline memory encoding: document-wise RoPE + chunk-mean pooling
// (MSA, b-lab.team summary, stage "Global Memory Encoding" and item 1
// "Document-wise RoPE"; Evermind summary sec. 2, fixed-length chunks with
// mean pooling).
//
// One CTA pools one chunk of one array.  Thread i owns 4 consecutive elements
// of the [heads][dim] row (for K: 4 rotate-half pairs, i.e. 4 elements of the
// first half and their 4 partners), walks the chunk's tokens and adds them with
// a fixed pairwise tree of 64 leaves (absent tokens of a short chunk are exact
// zeros).  The tree depends only on the token's place inside its chunk, and
// chunks are cut relative to the document start, so a document encoded alone
// gives the same bytes as inside the memory.
#pragma once
#include "common.cuh"

namespace msa {

struct ChunkSpan {
  int64_t t0;  // first token (global index)
  int32_t n;   // tokens in the chunk
  int32_t p0;  // document-relative position of the first token
};

__device__ __forceinline__ ChunkSpan chunk_span(int64_t c, const int32_t *__restrict__ chunk_doc,
                                                const int64_t *__restrict__ doc_tok_off,
                                                const int64_t *__restrict__ doc_chunk_off,
                                                int L) {
  const int d = chunk_doc[c];
  const int64_t j = c - doc_chunk_off[d];
  const int64_t t0 = doc_tok_off[d] + j * L;
  const int64_t rem = doc_tok_off[d + 1] - t0;
  ChunkSpan s;
  s.t0 = t0;
  s.n = static_cast<int32_t>(rem < L ? rem : L);
  s.p0 = static_cast<int32_t>(j * L);
  return s;
}

// Binary-counter pairwise summation: leaf t merges with the pending partial
// sums of every level whose bit is set in t.  After leaf 63, s[6] holds the
// total of all 64 leaves (a balanced tree of depth 6).
template <int E>
__device__ __forceinline__ void tree_push(float (&s)[7][E], float (&x)[E], const int t) {
#pragma unroll
  for (int lvl = 0; lvl < 6; ++lvl) {
    if (t & (1 << lvl)) {
#pragma unroll
      for (int e = 0; e < E; ++e) x[e] = s[lvl][e] + x[e];
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) s[lvl][e] = x[e];
      return;
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) s[6][e] = x[e];
}

// V and router keys: plain chunk mean.  NORMALIZE additionally divides each
// router head by max(|mean|, eps) (stored unit router keys).
//   X       : token-major rows of width W (= heads * dim); row 0 = token tok_base
//   out     : chunk c's result at out + c * out_stride + out_off
//   mean_out: optional un-normalised means [C][W]
template <typename T, bool NORMALIZE>
__global__ void __launch_bounds__(1024)
pool_plain_kernel(const T *__restrict__ X, int64_t tok_base, int W, int64_t c_begin,
                  const int32_t *__restrict__ chunk_doc, const int64_t *__restrict__ doc_tok_off,
                  const int64_t *__restrict__ doc_chunk_off, int L, T *__restrict__ out,
                  int64_t out_stride, int64_t out_off, int head_dim, T *__restrict__ mean_out) {
  const int64_t c = c_begin + blockIdx.x;
  const ChunkSpan sp = chunk_span(c, chunk_doc, doc_tok_off, doc_chunk_off, L);
  const int e0 = threadIdx.x * 4;
  const bool active = e0 < W;
  const T *src = X + (sp.t0 - tok_base) * static_cast<int64_t>(W) + (active ? e0 : 0);

  float s[7][4];
  // Leaves in batches of 8 so that several loads are in flight per thread.
#pragma unroll
  for (int tb = 0; tb < kMaxChunkLen; tb += 8) {
    float xb[8][4];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (active && tb + u < sp.n) {
        load4(src + static_cast<int64_t>(tb + u) * W, xb[u]);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) xb[u][e] = 0.0f;
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) tree_push<4>(s, xb[u], tb + u);
  }
  float m[4];
  const float n = static_cast<float>(sp.n);
#pragma unroll
  for (int e = 0; e < 4; ++e) m[e] = __fdiv_rn(s[6][e], n);

  if (mean_out != nullptr && active) store4(mean_out + c * W + e0, m);
  if (NORMALIZE) {
    // threads of one head are an aligned power-of-two group inside a warp
    float ss = 0.0f;
#pragma unroll
    for (int e = 0; e < 4; ++e) ss = fmaf(m[e], m[e], ss);
    const int group = head_dim / 4;
    for (int o = group / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = 1.0f / fmaxf(sqrtf(ss), kEps);
#pragma unroll
    for (int e = 0; e < 4; ++e) m[e] *= inv;
  }
  if (active) store4(out + c * out_stride + out_off + e0, m);
}

// K: rotate every token at its document-relative position, then pool.
// Thread i handles head h = i / (D/8) and pairs [4q, 4q+4) with
// q = i % (D/8): elements 4q.. and their partners 4q + D/2.. .
//   rope: [rope_len][D/2] (cos, sin) of position * theta^(-2i/D)
template <typename T>
__global__ void __launch_bounds__(1024)
pool_rope_kernel(const T *__restrict__ K, int64_t tok_base, int H, int D, int64_t c_begin,
                 const int32_t *__restrict__ chunk_doc, const int64_t *__restrict__ doc_tok_off,
                 const int64_t *__restrict__ doc_chunk_off, int L, const float2 *__restrict__ rope,
                 T *__restrict__ out, int64_t out_stride) {
  const int64_t c = c_begin + blockIdx.x;
  const ChunkSpan sp = chunk_span(c, chunk_doc, doc_tok_off, doc_chunk_off, L);
  const int per_head = D / 8;
  const int h = threadIdx.x / per_head;
  const int i0 = (threadIdx.x % per_head) * 4;
  const bool active = h < H;
  const int W = H * D;
  const int half = D / 2;
  const T *src = K + (sp.t0 - tok_base) * static_cast<int64_t>(W) + (active ? h * D + i0 : 0);

  float s[7][8];
#pragma unroll
  for (int tb = 0; tb < kMaxChunkLen; tb += 4) {
    float xb[4][8];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = tb + u;
      if (active && t < sp.n) {
        float a[4], b[4];
        load4(src + static_cast<int64_t>(t) * W, a);
        load4(src + static_cast<int64_t>(t) * W + half, b);
        const float2 *cs = rope + static_cast<int64_t>(sp.p0 + t) * half + i0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 r = cs[e];
          xb[u][e] = a[e] * r.x - b[e] * r.y;
          xb[u][4 + e] = b[e] * r.x + a[e] * r.y;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) xb[u][e] = 0.0f;
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) tree_push<8>(s, xb[u], tb + u);
  }
  if (!active) return;
  const float n = static_cast<float>(sp.n);
  float lo[4], hi[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    lo[e] = __fdiv_rn(s[6][e], n);
    hi[e] = __fdiv_rn(s[6][4 + e], n);
  }
  T *dst = out + c * out_stride + h * D + i0;
  store4(dst, lo);
  store4(dst + half, hi);
}

}  // namespace msa
