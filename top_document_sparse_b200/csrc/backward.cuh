// backward.cuh -- gradients of the routing score and of the sparse attention,
// for training the router with an auxiliary routing loss and the model
// through the sparse context (MSA, Evermind summary sec. 4A: continued
// pre-training supervises routing with L_aux; b-lab.team item 1 and stage
// "Sparse Generation" for the attention being differentiated).
//
//   route_backward_kernel   one warp per (query, document) with a nonzero
//                           upstream gradient: recompute the document's
//                           score over every (token, chunk), take the first
//                           maximising pair (token, then chunk order), and
//                           scatter the cosine's gradient to that token's
//                           query row and that chunk's pooled router key
//   attend_backward_kernel  one warp per (query, token, query head): three
//                           passes over the token's context -- softmax
//                           statistics, the output O (for <dO, O>), then the
//                           gradients dq' (kept in registers, rotated back to
//                           dQ), and dkey / dvalue of every context row
//                           (atomic adds: rows are shared by the heads of a
//                           GQA group, by tokens and by queries)
// Both accumulate in fp32 from bf16 or fp32 inputs.  They favour plainness
// over speed (CUDA cores, no tiling).
#pragma once
#include "attend.cuh"
#include "common.cuh"

namespace msa {

// grid-stride over warps, block 256.  Qr [B][T][W], means [C][W] (the pooled,
// un-normalised router keys), G [B][n_docs]; dQr [B][T][W], dmeans [C][W]
// zeroed by the caller.  W = H_r * d_r.
template <typename T>
__global__ void __launch_bounds__(256)
route_backward_kernel(const T *__restrict__ Qr, int B, int T_tok, const T *__restrict__ means,
                      const int64_t *__restrict__ doc_chunk_off, int n_docs, int H_r, int d_r,
                      const float *__restrict__ G, float *__restrict__ dQr,
                      float *__restrict__ dmeans) {
  const int lane = threadIdx.x & 31;
  const int64_t W = static_cast<int64_t>(H_r) * d_r;
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * (blockDim.x / 32);
  for (int64_t p = blockIdx.x * static_cast<int64_t>(blockDim.x / 32) + threadIdx.x / 32;
       p < static_cast<int64_t>(B) * n_docs; p += n_warps) {
    const float g = G[p];
    if (g == 0.0f || T_tok < 1) continue;
    const int b = static_cast<int>(p / n_docs), d = static_cast<int>(p % n_docs);
    const int64_t c0 = doc_chunk_off[d], c1 = doc_chunk_off[d + 1];
    float best = -INFINITY;
    int tb = 0;
    int64_t cb = c0;
    for (int t = 0; t < T_tok; ++t) {
      const T *q = Qr + (static_cast<int64_t>(b) * T_tok + t) * W;
      for (int64_t c = c0; c < c1; ++c) {
        const T *k = means + c * W;
        float s = 0.0f;
        for (int h = 0; h < H_r; ++h) {
          float dot = 0.0f, qq = 0.0f, kk = 0.0f;
          for (int e = lane; e < d_r; e += 32) {
            const float a = Elem<T>::to_f(q[h * d_r + e]), bb = Elem<T>::to_f(k[h * d_r + e]);
            dot += a * bb;
            qq += a * a;
            kk += bb * bb;
          }
          dot = warp_sum(dot);
          qq = warp_sum(qq);
          kk = warp_sum(kk);
          s += dot / (fmaxf(sqrtf(qq), kEps) * fmaxf(sqrtf(kk), kEps));
        }
        s /= static_cast<float>(H_r);
        if (s > best) {  // strict: the first maximising pair
          best = s;
          tb = t;
          cb = c;
        }
      }
    }
    const T *q = Qr + (static_cast<int64_t>(b) * T_tok + tb) * W;
    const T *k = means + cb * W;
    float *dq = dQr + (static_cast<int64_t>(b) * T_tok + tb) * W;
    float *dk = dmeans + cb * W;
    const float gh = g / static_cast<float>(H_r);
    for (int h = 0; h < H_r; ++h) {
      float dot = 0.0f, qq = 0.0f, kk = 0.0f;
      for (int e = lane; e < d_r; e += 32) {
        const float a = Elem<T>::to_f(q[h * d_r + e]), bb = Elem<T>::to_f(k[h * d_r + e]);
        dot += a * bb;
        qq += a * a;
        kk += bb * bb;
      }
      dot = warp_sum(dot);
      qq = warp_sum(qq);
      kk = warp_sum(kk);
      const float rq = sqrtf(qq), rk = sqrtf(kk);
      const float nq = fmaxf(rq, kEps), nk = fmaxf(rk, kEps);
      const float cs = dot / (nq * nk);
      for (int e = lane; e < d_r; e += 32) {
        const float a = Elem<T>::to_f(q[h * d_r + e]), bb = Elem<T>::to_f(k[h * d_r + e]);
        float gq = bb / (nq * nk), gk = a / (nq * nk);
        if (rq >= kEps) gq -= cs * a / (nq * nq);  // a clamped norm is a constant
        if (rk >= kEps) gk -= cs * bb / (nk * nk);
        atomicAdd(dq + h * d_r + e, gh * gq);
        atomicAdd(dk + h * d_r + e, gh * gk);
      }
    }
  }
}

// grid (B * T), block H_q * 32: warp h owns query head h of token i of query
// b; a lane owns elements lane + 32 u of a head (rotate-half partners share a
// lane: D / 2 is a multiple of 32).  Context of token i: [memory rows of
// ids[b], rank order] ++ [local rows 0 .. j], j = cache_len0[b] + i, the keys
// as stored (pooled K after document-wise RoPE; local K after RoPE at
// pos_offset + l).  dQ [B][T][H_q][D] is written; d_content [C][2][H_kv][D]
// and d_cache_k / d_cache_v [B][cap][H_kv][D] are accumulated (zeroed by the
// caller), the key gradients with respect to the keys as stored.
template <typename T, int D>
__global__ void __launch_bounds__(1024)
attend_backward_kernel(const T *__restrict__ content, const int32_t *__restrict__ ids, int k,
                       const int64_t *__restrict__ doc_chunk_off, int n_docs, int H_kv, int H_q,
                       const T *__restrict__ Q, int T_tok, const T *__restrict__ K_cache,
                       const T *__restrict__ V_cache, const int32_t *__restrict__ cache_len0,
                       int cap, int pos_offset, const float2 *__restrict__ rope, float scale,
                       const T *__restrict__ dO, float *__restrict__ dQ,
                       float *__restrict__ d_content, float *__restrict__ d_cache_k,
                       float *__restrict__ d_cache_v) {
  constexpr int U = D / 32;
  __shared__ int table[kMaxMemRows];
  __shared__ int pre[kMaxTopK + 1];
  __shared__ int base[kMaxTopK];
  const int b = blockIdx.x / T_tok, i = blockIdx.x % T_tok;
  const int h = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_mem = build_chunk_table(ids + static_cast<int64_t>(b) * k, k, doc_chunk_off, n_docs,
                                      nullptr, 0, table, pre, base, kMaxMemRows);
  if (h >= H_q) return;
  const int j = cache_len0[b] + i;
  float *dq_out = dQ + ((static_cast<int64_t>(b) * T_tok + i) * H_q + h) * D;
  if (j >= cap || j < 0) {
    if (lane == 0 && h == 0) raise_device_error(MSA_DEVERR_CACHE_OVERFLOW);
    for (int u = 0; u < U; ++u) dq_out[lane + 32 * u] = 0.0f;
    return;
  }
  const int g = h / (H_q / H_kv);
  const int half = D / 2;
  const float2 *cs = rope + static_cast<int64_t>(pos_offset + j) * half;
  float q[U], go[U];
  {
    const T *qs = Q + ((static_cast<int64_t>(b) * T_tok + i) * H_q + h) * D;
    const T *gs = dO + ((static_cast<int64_t>(b) * T_tok + i) * H_q + h) * D;
    float x[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      x[u] = Elem<T>::to_f(qs[lane + 32 * u]);
      go[u] = Elem<T>::to_f(gs[lane + 32 * u]);
    }
#pragma unroll
    for (int u = 0; u < U / 2; ++u) {
      const float2 r = cs[lane + 32 * u];
      q[u] = x[u] * r.x - x[u + U / 2] * r.y;
      q[u + U / 2] = x[u + U / 2] * r.x + x[u] * r.y;
    }
  }
  const int n_ctx = n_mem + j + 1;
  const int64_t kv = static_cast<int64_t>(H_kv) * D;
  auto rows = [&](int x, const T *&kr, const T *&vr, float *&dk, float *&dv) {
    if (x < n_mem) {
      const int64_t row = static_cast<int64_t>(table[x]) * 2 * kv + g * D;
      kr = content + row;
      vr = kr + kv;
      dk = d_content + row;
      dv = dk + kv;
    } else {
      const int64_t row = (static_cast<int64_t>(b) * cap + (x - n_mem)) * kv + g * D;
      kr = K_cache + row;
      vr = V_cache + row;
      dk = d_cache_k + row;
      dv = d_cache_v + row;
    }
  };
  auto logit = [&](const T *kr) {
    float dot = 0.0f;
#pragma unroll
    for (int u = 0; u < U; ++u) dot = fmaf(q[u], Elem<T>::to_f(kr[lane + 32 * u]), dot);
    return warp_sum(dot) * scale;
  };
  // pass 1: softmax statistics
  float m = -INFINITY, l = 0.0f;
  for (int x = 0; x < n_ctx; ++x) {
    const T *kr, *vr;
    float *dk, *dv;
    rows(x, kr, vr, dk, dv);
    const float z = logit(kr);
    const float mn = fmaxf(m, z);
    l = l * expf(m - mn) + expf(z - mn);
    m = mn;
  }
  const float inv_l = 1.0f / l;
  // pass 2: O, then Dv = <dO, O>
  float o[U];
#pragma unroll
  for (int u = 0; u < U; ++u) o[u] = 0.0f;
  for (int x = 0; x < n_ctx; ++x) {
    const T *kr, *vr;
    float *dk, *dv;
    rows(x, kr, vr, dk, dv);
    const float p = expf(logit(kr) - m) * inv_l;
#pragma unroll
    for (int u = 0; u < U; ++u) o[u] = fmaf(p, Elem<T>::to_f(vr[lane + 32 * u]), o[u]);
  }
  float dv_dot = 0.0f;
#pragma unroll
  for (int u = 0; u < U; ++u) dv_dot = fmaf(go[u], o[u], dv_dot);
  dv_dot = warp_sum(dv_dot);
  // pass 3: gradients
  float dq[U];
#pragma unroll
  for (int u = 0; u < U; ++u) dq[u] = 0.0f;
  for (int x = 0; x < n_ctx; ++x) {
    const T *kr, *vr;
    float *dk, *dv;
    rows(x, kr, vr, dk, dv);
    const float p = expf(logit(kr) - m) * inv_l;
    float dp = 0.0f;
#pragma unroll
    for (int u = 0; u < U; ++u) dp = fmaf(go[u], Elem<T>::to_f(vr[lane + 32 * u]), dp);
    dp = warp_sum(dp);
    const float dz = p * (dp - dv_dot) * scale;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      dq[u] = fmaf(dz, Elem<T>::to_f(kr[lane + 32 * u]), dq[u]);
      atomicAdd(dk + lane + 32 * u, dz * q[u]);
      atomicAdd(dv + lane + 32 * u, p * go[u]);
    }
  }
  // dQ = the rotation's transpose applied to dq'
#pragma unroll
  for (int u = 0; u < U / 2; ++u) {
    const float2 r = cs[lane + 32 * u];
    dq_out[lane + 32 * u] = dq[u] * r.x + dq[u + U / 2] * r.y;
    dq_out[lane + 32 * (u + U / 2)] = dq[u + U / 2] * r.x - dq[u] * r.y;
  }
}

}  // namespace msa
