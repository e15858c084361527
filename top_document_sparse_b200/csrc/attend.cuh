// attend.cuh -- sparse generation (MSA, b-lab.team summary item 1 "Scalable
// Sparse Attention" and "Global RoPE", stage "Sparse Generation"):
// the new tokens attend over [pooled K/V of the retrieved documents' chunks,
// rank order, all visible] ++ [local cache rows 0..j, causal], with Q and the
// new K rotated at pos_offset + j.
//
// Kernels:
//   append_kernel         rotate the new K rows, write K/V into the local cache
//   attend_simt_kernel    fp32 path (CUDA cores, one warp per query head)
//   attend_mma_kernel     bf16 one-token (decode) path: per (query, kv head,
//                         context split) CTA, 3 warps stream 16-row context
//                         blocks (cp.async, double-buffered, XOR-swizzled
//                         smem) and run S^T = K Q^T and O^T += V^T P^T on
//                         mma.sync with an online softmax (context rows / head
//                         dim on M, the GQA group's heads on N)
//   attend_combine_kernel merge context splits (log-sum-exp) and advance
//                         cache_len (a one-split decode call advances it in
//                         the attention kernel, whose CTAs of one query form
//                         a cluster)
//   attend_prefill_kernel bf16 calls of more than one token: per (query, kv
//                         head, tile of 64 / G tokens) CTA, the tile's query
//                         rows on M and each staged context block shared by
//                         its four warps (see below)
//   advance_kernel        cache_len += tokens where no kernel above does it
// For a one-token call (decode) the attention kernel appends the new row
// itself; longer calls run append_kernel first.
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace msa {

constexpr int kMaxMemRows = 4096;  // retrieved chunks per query (k * chunks per doc)
constexpr float kLog2e = 1.4426950408889634f;

// Chunk list of query b's retrieved documents in rank order -> table[0..n_mem).
// Warp 0 loads the k (<= 64) ranks' chunk counts in parallel (two ranks per
// lane) and prefix-sums them with shuffles; every thread then fills table
// entries from shared memory only (binary search over the prefix sums).
// Ids outside [0, n_docs) contribute no rows and raise MSA_DEVERR_BAD_DOC_ID.
// slots_b (nullable, [k]): chunk rows of rank r start at slots_b[r] *
// slot_chunks instead of doc_chunk_off[id] (device slot cache of a host tier).
// `pre` needs kMaxTopK + 1 ints and `base` kMaxTopK ints of shared memory.
__device__ __forceinline__ int build_chunk_table(const int32_t *__restrict__ ids_b, int k,
                                                 const int64_t *__restrict__ doc_chunk_off,
                                                 int n_docs, const int32_t *__restrict__ slots_b,
                                                 int slot_chunks, int *table, int *pre,
                                                 int *base, int table_cap) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int cnt[2] = {0, 0};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = lane + 32 * h;
      if (r < k) {
        const int d = ids_b[r];
        if (d >= 0 && d < n_docs) {
          const int64_t c0 = doc_chunk_off[d];
          cnt[h] = static_cast<int>(doc_chunk_off[d + 1] - c0);
          base[r] = slots_b ? slots_b[r] * slot_chunks : static_cast<int>(c0);
        } else {
          raise_device_error(MSA_DEVERR_BAD_DOC_ID);
          base[r] = 0;
        }
      }
    }
    int run = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      int v = cnt[h];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      const int r = lane + 32 * h;
      const int excl = run + v - cnt[h];
      // a rank that would overflow the table contributes nothing (host validation keeps
      // k * max_doc_chunks <= table_cap, so this does not happen)
      if (r < k) pre[r] = excl + cnt[h] > table_cap ? min(excl, table_cap) : excl;
      run += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) pre[k] = min(run, table_cap);
  }
  __syncthreads();
  const int n_mem = pre[k];
  for (int x = threadIdx.x; x < n_mem; x += blockDim.x) {
    int lo = 0, hi = k - 1;  // last rank r with pre[r] <= x
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pre[mid] <= x) lo = mid; else hi = mid - 1;
    }
    table[x] = base[lo] + (x - pre[lo]);
  }
  __syncthreads();
  return n_mem;
}

// ---------------------------------------------------------------- append
// grid (B * T); thread i handles head h = i / (D/8) and the rotate-half pairs
// [4q, 4q+4) of that head (K) plus 8 elements of V.
template <typename T>
__global__ void append_kernel(const T *__restrict__ K_new, const T *__restrict__ V_new, int T_tok,
                              int H_kv, int D, T *__restrict__ K_cache, T *__restrict__ V_cache,
                              const int32_t *__restrict__ cache_len, int cap, int pos_offset,
                              const float2 *__restrict__ rope) {
  const int b = blockIdx.x / T_tok, i = blockIdx.x % T_tok;
  const int j = cache_len[b] + i;
  if (j >= cap || j < 0) {
    if (threadIdx.x == 0) raise_device_error(MSA_DEVERR_CACHE_OVERFLOW);
    return;
  }
  const int per_head = D / 8;
  const int h = threadIdx.x / per_head;
  if (h >= H_kv) return;
  const int i0 = (threadIdx.x % per_head) * 4;
  const int half = D / 2;
  const int64_t src = (static_cast<int64_t>(b) * T_tok + i) * H_kv * D + h * D;
  const int64_t dst = (static_cast<int64_t>(b) * cap + j) * H_kv * D + h * D;
  float a[4], c[4], lo[4], hi[4];
  load4(K_new + src + i0, a);
  load4(K_new + src + half + i0, c);
  const float2 *cs = rope + static_cast<int64_t>(pos_offset + j) * half + i0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 r = cs[e];
    lo[e] = a[e] * r.x - c[e] * r.y;
    hi[e] = c[e] * r.x + a[e] * r.y;
  }
  store4(K_cache + dst + i0, lo);
  store4(K_cache + dst + half + i0, hi);
  float v[4];
  load4(V_new + src + i0, v);
  store4(V_cache + dst + i0, v);
  load4(V_new + src + half + i0, v);
  store4(V_cache + dst + half + i0, v);
}

// ---------------------------------------------------------------- fp32 path
// grid (B * T), block H_q * 32: warp h owns query head h; lane owns the
// elements lane + 32u of the head (a rotate-half partner lives in the same
// lane because D/2 is a multiple of 32).
template <typename T, int D>
__global__ void __launch_bounds__(512)
attend_simt_kernel(const T *__restrict__ content, const int32_t *__restrict__ ids, int k,
                   const int64_t *__restrict__ doc_chunk_off, int n_docs,
                   const int32_t *__restrict__ slots, int slot_chunks, int H_kv, int H_q,
                   const T *__restrict__ Q, int T_tok, const T *__restrict__ K_cache,
                   const T *__restrict__ V_cache, const int32_t *__restrict__ cache_len, int cap,
                   int pos_offset, const float2 *__restrict__ rope, float scale,
                   T *__restrict__ O) {
  constexpr int U = D / 32;
  __shared__ int table[kMaxMemRows];
  __shared__ int pre[kMaxTopK + 1];
  __shared__ int base[kMaxTopK];
  const int b = blockIdx.x / T_tok, i = blockIdx.x % T_tok;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_mem = build_chunk_table(ids + static_cast<int64_t>(b) * k, k, doc_chunk_off, n_docs,
                                      slots ? slots + static_cast<int64_t>(b) * k : nullptr,
                                      slot_chunks, table, pre, base, kMaxMemRows);
  const int j = cache_len[b] + i;
  const int h = warp;
  if (h >= H_q) return;
  T *out = O + ((static_cast<int64_t>(b) * T_tok + i) * H_q + h) * D;
  if (j >= cap) {  // the append kernel has flagged the overflow
    for (int u = 0; u < U; ++u) out[lane + 32 * u] = Elem<T>::from_f(0.0f);
    return;
  }
  const int g = h / (H_q / H_kv);
  const int half = D / 2;
  float q[U];
  {
    const T *qs = Q + ((static_cast<int64_t>(b) * T_tok + i) * H_q + h) * D;
    float x[U];
#pragma unroll
    for (int u = 0; u < U; ++u) x[u] = Elem<T>::to_f(qs[lane + 32 * u]);
    const float2 *cs = rope + static_cast<int64_t>(pos_offset + j) * half;
#pragma unroll
    for (int u = 0; u < U / 2; ++u) {
      const float2 r = cs[lane + 32 * u];
      q[u] = x[u] * r.x - x[u + U / 2] * r.y;
      q[u + U / 2] = x[u + U / 2] * r.x + x[u] * r.y;
    }
  }
  float m = -INFINITY, l = 0.0f, acc[U];
#pragma unroll
  for (int u = 0; u < U; ++u) acc[u] = 0.0f;
  const int n_ctx = n_mem + j + 1;
  const int64_t kv = static_cast<int64_t>(H_kv) * D;
  for (int x = 0; x < n_ctx; ++x) {
    const T *kr, *vr;
    if (x < n_mem) {
      kr = content + static_cast<int64_t>(table[x]) * 2 * kv + g * D;
      vr = kr + kv;
    } else {
      const int64_t row = (static_cast<int64_t>(b) * cap + (x - n_mem)) * kv + g * D;
      kr = K_cache + row;
      vr = V_cache + row;
    }
    float dot = 0.0f;
#pragma unroll
    for (int u = 0; u < U; ++u) dot = fmaf(q[u], Elem<T>::to_f(kr[lane + 32 * u]), dot);
    dot = warp_sum(dot) * scale;
    const float m_new = fmaxf(m, dot);
    const float alpha = expf(m - m_new);
    const float p = expf(dot - m_new);
    l = l * alpha + p;
#pragma unroll
    for (int u = 0; u < U; ++u) acc[u] = fmaf(p, Elem<T>::to_f(vr[lane + 32 * u]), acc[u] * alpha);
    m = m_new;
  }
  const float inv = 1.0f / l;
#pragma unroll
  for (int u = 0; u < U; ++u) out[lane + 32 * u] = Elem<T>::from_f(acc[u] * inv);
}

// ---------------------------------------------------------------- bf16 path
// Three warps per CTA: 3 x 2 stages x 2 x 16 x D x 2 B of ring (48 KB at D = 128) lets four
// CTAs share an SM, so the 8 x 64 (query, kv head) CTAs of a decode batch run in one wave.
constexpr int kAttWarps = 3;
constexpr int kAttRows = 16;  // context rows per warp block
// Early path: local blocks past the ring's first that a warp may prefetch into
// L2 while the previous kernel (the top-k) finishes.  None by default: measured
// on the 1M decode once the query normalisation ran before its dependency wait,
// 1,543 steps/s with none, 1,494 with two blocks, 1,475 with four.
#ifndef MSA_ATT_EARLY_L2
#define MSA_ATT_EARLY_L2 0
#endif
constexpr int kAttEarlyL2 = MSA_ATT_EARLY_L2;

template <int D>
struct AttSmem {
  static constexpr int kBlockBytes = kAttRows * D * 2;       // one K or V block
  static constexpr int kWarpBytes = 2 /*stages*/ * 2 /*K,V*/ * kBlockBytes;
  static constexpr int kQBytes = 16 * D * 2;
  static constexpr int kMergeBytes = kAttWarps * 16 * (D + 2) * 4;
  static constexpr int kRing = kAttWarps * kWarpBytes;
  static constexpr int kFixed =
      (kRing > kMergeBytes ? kRing : kMergeBytes) + kQBytes + (2 * kMaxTopK + 1) * 4;
  static int bytes(int table_cap) { return kFixed + table_cap * 4; }
};

// Byte offset of 16-byte chunk `c` of row `r` in a [rows][D] bf16 tile whose
// chunks are XOR-swizzled by (r & 7) (conflict-free ldmatrix).
template <int D>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return static_cast<uint32_t>(r * (D * 2) + ((c ^ (r & 7)) << 4));
}

// grid (B * H_kv, n_split, T), block 32 * kAttWarps.
template <int D, int G>
__global__ void __launch_bounds__(32 * kAttWarps)
attend_mma_kernel(const __nv_bfloat16 *__restrict__ content, const int32_t *__restrict__ ids,
                  int k, const int64_t *__restrict__ doc_chunk_off, int n_docs,
                  const int32_t *__restrict__ slots, int slot_chunks, int H_kv,
                  const __nv_bfloat16 *__restrict__ Q, int T_tok,
                  __nv_bfloat16 *__restrict__ K_cache, __nv_bfloat16 *__restrict__ V_cache,
                  const __nv_bfloat16 *__restrict__ K_new, const __nv_bfloat16 *__restrict__ V_new,
                  int32_t *__restrict__ cache_len, int cap, int pos_offset,
                  const float2 *__restrict__ rope, float scale_log2, int n_split, int table_cap,
                  int fuse_append, int early, int cluster_advance, __nv_bfloat16 *__restrict__ O,
                  float *__restrict__ part_o, float *__restrict__ part_ml) {
  constexpr int CPR = D / 8;  // 16-byte chunks per row
  using Sm = AttSmem<D>;
  extern __shared__ __align__(128) uint8_t sm[];
  uint8_t *ring = sm;
  uint8_t *qsm = sm + (Sm::kRing > Sm::kMergeBytes ? Sm::kRing : Sm::kMergeBytes);
  int *pre = reinterpret_cast<int *>(qsm + Sm::kQBytes);
  int *base = pre + (kMaxTopK + 1);
  int *table = base + kMaxTopK;

  const int H_q = H_kv * G;
  const int b = blockIdx.x / H_kv, g = blockIdx.x % H_kv;
  const int split = blockIdx.y, i = blockIdx.z;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t kv = static_cast<int64_t>(H_kv) * D;
  const int half = D / 2;
  // Context order: [local rows 0..j (causal) | memory rows in rank order]; the
  // softmax does not depend on it.  The local part needs only cache_len, Q,
  // the new token and the local cache, not the retrieved ids: with `early`
  // (the caller guarantees that the kernel before this one on the stream
  // writes none of those) and one split, the CTA starts on it before waiting
  // for the previous kernel, reading them through L2.
  const bool early_ok = early && n_split == 1;
  if (!early_ok) {
    griddep_wait();
    griddep_launch();
  }
  const int j = (early_ok ? __ldcg(cache_len + b) : cache_len[b]) + i;
  // cluster_advance (one token, one split, launched as clusters of the query's
  // H_kv CTAs): this CTA has read cache_len; rank 0 advances it at the end,
  // after every CTA of the cluster has arrived here
  if (cluster_advance) asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  const bool overflow = j >= cap || j < 0;
  const int n_loc = overflow ? 0 : j + 1;
  int n_mem = 0, x0 = 0, x1 = n_loc;  // until the table is built, only local rows are issued

  // one-token call: the CTA whose range holds the new row (local row j)
  // rotates K_new at pos_offset + j and writes K and V to the cache before any
  // of its copies can read that row
  auto append_new_row = [&]() {
    const int64_t src = static_cast<int64_t>(b) * kv + g * D;
    const int64_t dst = (static_cast<int64_t>(b) * cap + j) * kv + g * D;
    const float2 *cs = rope + static_cast<int64_t>(pos_offset + j) * half;
    for (int e = threadIdx.x; e < half; e += blockDim.x) {
      const float a = __bfloat162float(__ldcg(K_new + src + e));
      const float c = __bfloat162float(__ldcg(K_new + src + e + half));
      const float2 t = cs[e];
      K_cache[dst + e] = __float2bfloat16_rn(a * t.x - c * t.y);
      K_cache[dst + e + half] = __float2bfloat16_rn(c * t.x + a * t.y);
      V_cache[dst + e] = __ldcg(V_new + src + e);
      V_cache[dst + e + half] = __ldcg(V_new + src + e + half);
    }
    __threadfence();  // the row is read back through cp.async (L2)
    __syncthreads();
  };
  if (fuse_append && overflow && threadIdx.x == 0 && g == 0 && split == 0)
    raise_device_error(MSA_DEVERR_CACHE_OVERFLOW);
  if (early_ok && fuse_append && !overflow) append_new_row();  // one split holds every row

  uint8_t *wbuf = ring + warp * Sm::kWarpBytes;
  // issue the loads of the block starting at context row x into stage s
  auto issue = [&](int x, int s) {
    uint8_t *kb = wbuf + s * 2 * Sm::kBlockBytes;
    uint8_t *vb = kb + Sm::kBlockBytes;
#pragma unroll
    for (int u = 0; u < kAttRows * CPR / 32; ++u) {
      const int idx = lane + 32 * u;
      const int r = idx / CPR, c = idx % CPR;
      const int xr = x + r;
      const __nv_bfloat16 *ks = K_cache, *vs = V_cache;
      bool ok = xr < x1;
      if (ok) {
        if (xr < n_loc) {
          const int64_t row = (static_cast<int64_t>(b) * cap + xr) * kv + g * D;
          ks = K_cache + row;
          vs = V_cache + row;
        } else {
          ks = content + static_cast<int64_t>(table[xr - n_loc]) * 2 * kv + g * D;
          vs = ks + kv;
        }
      }
      cp_async_16(smem_u32(kb + swz<D>(r, c)), ks + c * 8, ok);
      cp_async_16(smem_u32(vb + swz<D>(r, c)), vs + c * 8, ok);
    }
    cp_async_commit();
  };
  // early: the first block of every warp is in flight before the wait if it is all local
  bool issued = false;
  if (early_ok && (warp + 1) * kAttRows <= n_loc) {
    issue(warp * kAttRows, 0);
    issued = true;
    // and the warp's next all-local blocks into L2: lane l takes row l / 2 of K (l even) or V
#pragma unroll 1
    for (int p = 1; p <= kAttEarlyL2; ++p) {
      const int x = (warp + p * kAttWarps) * kAttRows;
      if (x + kAttRows > n_loc) break;
      const __nv_bfloat16 *src = ((lane & 1) ? V_cache : K_cache) +
                                 (static_cast<int64_t>(b) * cap + x + (lane >> 1)) * kv + g * D;
#pragma unroll
      for (int o = 0; o < D * 2; o += 128) prefetch_l2(reinterpret_cast<const uint8_t *>(src) + o);
    }
  }
  // rotated query rows of the group -> qsm [16][D] (rows >= G are zero)
  {
    const __nv_bfloat16 *qb = Q + ((static_cast<int64_t>(b) * T_tok + i) * H_q + g * G) * D;
    const float2 *cs = rope + static_cast<int64_t>(pos_offset + (overflow ? 0 : j)) * half;
    for (int p = threadIdx.x; p < 16 * half; p += blockDim.x) {
      const int r = p / half, e = p % half;
      float lo = 0.0f, hi = 0.0f;
      if (r < G) {
        const float a = __bfloat162float(__ldcg(qb + r * D + e));
        const float c = __bfloat162float(__ldcg(qb + r * D + e + half));
        const float2 t = cs[e];
        lo = a * t.x - c * t.y;
        hi = c * t.x + a * t.y;
      }
      const __nv_bfloat16 blo = __float2bfloat16_rn(lo), bhi = __float2bfloat16_rn(hi);
      *reinterpret_cast<__nv_bfloat16 *>(qsm + swz<D>(r, e / 8) + (e % 8) * 2) = blo;
      *reinterpret_cast<__nv_bfloat16 *>(qsm + swz<D>(r, (e + half) / 8) + (e % 8) * 2) = bhi;
    }
  }
  if (early_ok) {
    griddep_wait();
    griddep_launch();
  }
  n_mem = build_chunk_table(ids + static_cast<int64_t>(b) * k, k, doc_chunk_off, n_docs,
                            slots ? slots + static_cast<int64_t>(b) * k : nullptr, slot_chunks,
                            table, pre, base, table_cap);
  const int n_ctx = overflow ? 0 : n_loc + n_mem;
  int per = (n_ctx + n_split - 1) / n_split;
  per = (per + kAttRows - 1) / kAttRows * kAttRows;
  x0 = split * per;
  x1 = min(n_ctx, x0 + per);
  if (!early_ok && fuse_append && !overflow && x0 <= j && j < x1) append_new_row();

  const int nblk = (x1 > x0) ? (x1 - x0 + kAttRows - 1) / kAttRows : 0;
  int s = 0;
  if (!issued && warp < nblk) issue(x0 + warp * kAttRows, 0);
  __syncthreads();

  // Transposed tile: S^T = K Q^T (M = 16 context rows, N = 8 heads per n tile,
  // K = D) and O^T += V^T P^T (M = D, N = heads, K = 16 context rows), P^T
  // reaching the B operand through movmatrix, so no MMA row is spent on the
  // GQA group's few heads.  A thread's accumulators hold heads
  // nt * 8 + (lane & 3) * 2 + {0, 1} and rows d = dm * 16 + lane / 4 (+ 8);
  // the online softmax state of a head is uniform over the 8 lane groups.
  constexpr int NT = (G + 7) / 8;  // n8 tiles of heads
  uint32_t qb[NT][D / 16][2];      // B fragments of Q^T (query rows >= G are zero)
  {
    const uint32_t qbase = smem_u32(qsm);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int kp = 0; kp < D / 32; ++kp)
        ldsm_x4(qbase + swz<D>(nt * 8 + (lane & 7), 4 * kp + (lane >> 3)), qb[nt][2 * kp][0],
                qb[nt][2 * kp][1], qb[nt][2 * kp + 1][0], qb[nt][2 * kp + 1][1]);
  }

  float mh[NT][2], lh[NT][2];  // running max (log2 units) and partial sum per head
  float acc[NT][D / 16][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    mh[nt][0] = mh[nt][1] = -INFINITY;
    lh[nt][0] = lh[nt][1] = 0.0f;
#pragma unroll
    for (int dm = 0; dm < D / 16; ++dm)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nt][dm][e] = 0.0f;
  }

  for (int bi = warp; bi < nblk; bi += kAttWarps) {
    const int x = x0 + bi * kAttRows;
    if (bi + kAttWarps < nblk) {
      issue(x + kAttWarps * kAttRows, s ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();
    const uint32_t kb = smem_u32(wbuf + s * 2 * Sm::kBlockBytes);
    const uint32_t vb = kb + Sm::kBlockBytes;

    // S^T = K Q^T over the block's 16 context rows
    float sc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[nt][e] = 0.0f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(kb + swz<D>(lane & 15, 2 * kk + (lane >> 4)), a0, a1, a2, a3);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        mma_bf16_16816(sc[nt], a0, a1, a2, a3, qb[nt][kk][0], qb[nt][kk][1]);
    }
    // online softmax per head over context rows x + lane/4 (c0, c1) and + 8 (c2, c3),
    // in log2 units; rows past the split end are masked
    const bool v0 = x + (lane >> 2) < x1, v1 = x + (lane >> 2) + 8 < x1;
    uint32_t pb[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float al[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float s0 = v0 ? sc[nt][h] * scale_log2 : -INFINITY;
        const float s1 = v1 ? sc[nt][2 + h] * scale_log2 : -INFINITY;
        float bm = fmaxf(s0, s1);
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
        const float mn = fmaxf(mh[nt][h], bm);  // finite: every block has a context row
        al[h] = exp2f(mh[nt][h] - mn);
        mh[nt][h] = mn;
        sc[nt][h] = exp2f(s0 - mn);
        sc[nt][2 + h] = exp2f(s1 - mn);
        lh[nt][h] = lh[nt][h] * al[h] + sc[nt][h] + sc[nt][2 + h];
      }
#pragma unroll
      for (int dm = 0; dm < D / 16; ++dm) {
        acc[nt][dm][0] *= al[0];
        acc[nt][dm][1] *= al[1];
        acc[nt][dm][2] *= al[0];
        acc[nt][dm][3] *= al[1];
      }
      // P^T as the B operand: transpose the two 8x8 bf16 quadrants in registers
      pb[nt][0] = movmatrix_trans(pack_bf16x2(sc[nt][0], sc[nt][1]));
      pb[nt][1] = movmatrix_trans(pack_bf16x2(sc[nt][2], sc[nt][3]));
    }
    // O^T += V^T P^T
#pragma unroll
    for (int dm = 0; dm < D / 16; ++dm) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4_trans(vb + swz<D>((lane & 7) + ((lane >> 4) << 3), 2 * dm + ((lane >> 3) & 1)), a0,
                    a1, a2, a3);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        mma_bf16_16816(acc[nt][dm], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
    }
    __syncwarp();
    s ^= 1;
  }

  // per-head totals over the 8 lane groups; the warps merge through shared memory
  __syncthreads();  // every warp is done with the ring: reuse it for the merge
  float *mo = reinterpret_cast<float *>(ring);  // [warp][16][D + 2]: D outputs, m, l
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float L = lh[nt][h];
      L += __shfl_xor_sync(0xffffffffu, L, 4);
      L += __shfl_xor_sync(0xffffffffu, L, 8);
      L += __shfl_xor_sync(0xffffffffu, L, 16);
      const int head = nt * 8 + (lane & 3) * 2 + h;
      float *row = mo + (warp * 16 + head) * (D + 2);
#pragma unroll
      for (int dm = 0; dm < D / 16; ++dm) {
        row[dm * 16 + (lane >> 2)] = acc[nt][dm][h];
        row[dm * 16 + (lane >> 2) + 8] = acc[nt][dm][2 + h];
      }
      if (lane < 4) {
        row[D] = mh[nt][h];
        row[D + 1] = L;
      }
    }
  __syncthreads();
  for (int p = threadIdx.x; p < G * D; p += blockDim.x) {
    const int r = p / D, e = p % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttWarps; ++w) M = fmaxf(M, mo[(w * 16 + r) * (D + 2) + D]);
    const float base = M == -INFINITY ? 0.0f : M;
    float L = 0.0f, acc_o = 0.0f;
#pragma unroll
    for (int w = 0; w < kAttWarps; ++w) {
      const float *row = mo + (w * 16 + r) * (D + 2);
      const float f = exp2f(row[D] - base);
      L += row[D + 1] * f;
      acc_o += row[e] * f;
    }
    const int h = g * G + r;
    const int64_t orow = (static_cast<int64_t>(b) * T_tok + i) * H_q + h;
    if (n_split == 1) {
      O[orow * D + e] = __float2bfloat16_rn(L > 0.0f ? acc_o / L : 0.0f);
    } else {
      part_o[(orow * n_split + split) * D + e] = acc_o;
      if (e == 0) {
        part_ml[(orow * n_split + split) * 2] = M;
        part_ml[(orow * n_split + split) * 2 + 1] = L;
      }
    }
  }
  if (cluster_advance) {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    if (g == 0 && threadIdx.x == 0) cache_len[b] = min(j + 1, cap);  // (i == 0: j is the old length)
  }
}

// grid (B * T * H_q), block D: merge the context splits.  Partial maxima are
// in log2 units.  The first block of each query also advances cache_len[b] by
// T (every attention CTA has read it by now).
__global__ void attend_combine_kernel(const float *__restrict__ part_o,
                                      const float *__restrict__ part_ml, int n_split, int D,
                                      __nv_bfloat16 *__restrict__ O, int32_t *__restrict__ cache_len,
                                      int rows_per_query, int T_tok, int cap) {
  griddep_wait();
  griddep_launch();
  const int64_t orow = blockIdx.x;
  if (threadIdx.x == 0 && orow % rows_per_query == 0) {
    int32_t *cl = cache_len + orow / rows_per_query;
    *cl = min(*cl + T_tok, cap);
  }
  const float *ml = part_ml + orow * n_split * 2;
  float M = -INFINITY;
  for (int s = 0; s < n_split; ++s) M = fmaxf(M, ml[2 * s]);
  const float base = M == -INFINITY ? 0.0f : M;
  for (int e = threadIdx.x; e < D; e += blockDim.x) {
    float L = 0.0f, acc = 0.0f;
    for (int s = 0; s < n_split; ++s) {
      const float f = exp2f(ml[2 * s] - base);
      L += ml[2 * s + 1] * f;
      acc += part_o[(orow * n_split + s) * D + e] * f;
    }
    O[orow * D + e] = __float2bfloat16_rn(L > 0.0f ? acc / L : 0.0f);
  }
}

__global__ void advance_kernel(int32_t *__restrict__ cache_len, int B, int T_tok, int cap) {
  griddep_wait();
  griddep_launch();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) cache_len[b] = min(cache_len[b] + T_tok, cap);
}

// ---------------------------------------------------------------- bf16 prefill
// Calls of more than one token: the FlashAttention-2 arrangement.  A warp owns
// 16 query rows -- 16 / G tokens x the GQA group's G heads -- with Q^T's
// fragments in registers; the CTA's four warps share every 32-row block of
// [memory rows in rank order | local rows 0..j_max] staged once in shared
// memory (two-stage cp.async ring), S = Q K^T and O += P V on mma.sync
// m16n8k16 with an online softmax per row (log2 units) and the causal mask
// j <= cache_len + t on local rows.  append_kernel has written the call's new
// rows before this kernel runs.  grid (B * H_kv, ceil(T / (4 * 16 / G))).
constexpr int kPfWarps = 4;
constexpr int kPfRows = 32;  // context rows per block

template <int D>
struct PfSmem {
  static constexpr int kBlockBytes = kPfRows * D * 2;  // one K or V block
  static constexpr int kRing = 2 /*stages*/ * 2 /*K,V*/ * kBlockBytes;
  static constexpr int kQBytes = kPfWarps * 16 * D * 2;
  static constexpr int kFixed = kRing + kQBytes + (2 * kMaxTopK + 1) * 4;
  static int bytes(int table_cap) { return kFixed + table_cap * 4; }
};

// (at most 128 registers: four CTAs per SM; measured 5% faster than three at 168)
template <int D, int G>
__global__ void __launch_bounds__(32 * kPfWarps, 4)
attend_prefill_kernel(const __nv_bfloat16 *__restrict__ content, const int32_t *__restrict__ ids,
                      int k, const int64_t *__restrict__ doc_chunk_off, int n_docs,
                      const int32_t *__restrict__ slots, int slot_chunks, int H_kv,
                      const __nv_bfloat16 *__restrict__ Q, int T_tok,
                      const __nv_bfloat16 *__restrict__ K_cache,
                      const __nv_bfloat16 *__restrict__ V_cache,
                      const int32_t *__restrict__ cache_len, int cap, int pos_offset,
                      const float2 *__restrict__ rope, float scale_log2, int table_cap,
                      __nv_bfloat16 *__restrict__ O) {
  static_assert(G >= 1 && G <= 16 && 16 % G == 0, "GQA group");
  constexpr int CPR = D / 8;         // 16-byte chunks per row
  constexpr int TW = 16 / G;         // tokens per warp
  constexpr int TC = kPfWarps * TW;  // tokens per CTA
  constexpr int NTD = D / 8;         // n8 tiles of the output row
  using Sm = PfSmem<D>;
  extern __shared__ __align__(128) uint8_t sm[];
  uint8_t *ring = sm;
  uint8_t *qsm = sm + Sm::kRing;
  int *pre = reinterpret_cast<int *>(qsm + Sm::kQBytes);
  int *base = pre + (kMaxTopK + 1);
  int *table = base + kMaxTopK;

  const int H_q = H_kv * G;
  const int b = blockIdx.x / H_kv, g = blockIdx.x % H_kv;
  const int t0 = blockIdx.y * TC;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t kv = static_cast<int64_t>(H_kv) * D;
  const int half = D / 2;
  griddep_wait();
  griddep_launch();
  const int len0 = cache_len[b];  // local rows before this call's tokens
  const int n_mem = build_chunk_table(ids + static_cast<int64_t>(b) * k, k, doc_chunk_off, n_docs,
                                      slots ? slots + static_cast<int64_t>(b) * k : nullptr,
                                      slot_chunks, table, pre, base, table_cap);
  const int t_last = min(t0 + TC, T_tok) - 1;  // last token of the tile
  const int n_loc = max(0, min(len0 + t_last + 1, cap));
  const int n_ctx = n_mem + n_loc;

  // rotated query rows -> qsm[warp][16][D]: row r = (token t0 + warp * TW + r / G, head
  // g * G + r % G); rows of tokens past the call are zero
  for (int p = threadIdx.x; p < kPfWarps * 16 * half; p += blockDim.x) {
    const int wr = p / (16 * half), r = (p / half) % 16, e = p % half;
    const int t = t0 + wr * TW + r / G;
    float lo = 0.0f, hi = 0.0f;
    if (t < T_tok && len0 + t < cap) {
      const __nv_bfloat16 *qr = Q + ((static_cast<int64_t>(b) * T_tok + t) * H_q + g * G + r % G) * D;
      const float a = __bfloat162float(qr[e]), c = __bfloat162float(qr[e + half]);
      const float2 cs = rope[static_cast<int64_t>(pos_offset + len0 + t) * half + e];
      lo = a * cs.x - c * cs.y;
      hi = c * cs.x + a * cs.y;
    }
    uint8_t *qw = qsm + wr * (16 * D * 2);
    *reinterpret_cast<__nv_bfloat16 *>(qw + swz<D>(r, e / 8) + (e % 8) * 2) = __float2bfloat16_rn(lo);
    *reinterpret_cast<__nv_bfloat16 *>(qw + swz<D>(r, (e + half) / 8) + (e % 8) * 2) =
        __float2bfloat16_rn(hi);
  }

  // the K and V rows of the block at context row x into stage st (one commit)
  auto issue = [&](int x, int st) {
    uint8_t *kb = ring + st * 2 * Sm::kBlockBytes;
#pragma unroll
    for (int u = 0; u < kPfRows * CPR * 2 / (32 * kPfWarps); ++u) {
      const int idx = threadIdx.x + 32 * kPfWarps * u;
      const int which = idx / (kPfRows * CPR), rem = idx % (kPfRows * CPR);
      const int r = rem / CPR, c = rem % CPR;
      const int xr = x + r;
      const bool ok = xr < n_ctx;
      const __nv_bfloat16 *src = which ? V_cache : K_cache;
      if (ok) {
        if (xr < n_mem)
          src = content + static_cast<int64_t>(table[xr]) * 2 * kv + which * kv + g * D;
        else
          src += (static_cast<int64_t>(b) * cap + (xr - n_mem)) * kv + g * D;
      }
      cp_async_16(smem_u32(kb + which * Sm::kBlockBytes + swz<D>(r, c)), src + c * 8, ok);
    }
    cp_async_commit();
  };
  const int nblk = (n_ctx + kPfRows - 1) / kPfRows;
  if (nblk > 0) issue(0, 0);
  __syncthreads();  // qsm complete

  // A fragments of this warp's 16 query rows
  uint32_t qa[D / 16][4];
  {
    const uint32_t qbase = smem_u32(qsm + warp * (16 * D * 2));
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
      ldsm_x4(qbase + swz<D>(lane & 15, 2 * kk + (lane >> 4)), qa[kk][0], qa[kk][1], qa[kk][2],
              qa[kk][3]);
  }
  // this thread's two rows: lane / 4 and lane / 4 + 8; the last context row each may see
  int vis[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int t = t0 + warp * TW + ((lane >> 2) + 8 * h) / G;
    vis[h] = n_mem + len0 + t;  // context index of local row len0 + t
  }
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.0f, 0.0f};
  float o[NTD][4];
#pragma unroll
  for (int nt = 0; nt < NTD; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[nt][e] = 0.0f;

  int st = 0;
  for (int blk = 0; blk < nblk; ++blk) {
    const int x = blk * kPfRows;
    if (blk + 1 < nblk) {
      issue(x + kPfRows, st ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // the block is in shared memory for every warp
    const uint32_t kb = smem_u32(ring + st * 2 * Sm::kBlockBytes);
    const uint32_t vb = kb + Sm::kBlockBytes;
    // S = Q K^T: 16 rows x 32 context columns (4 n8 tiles)
    float sc[kPfRows / 8][4];
#pragma unroll
    for (int nt = 0; nt < kPfRows / 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[nt][e] = 0.0f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
      for (int np = 0; np < kPfRows / 16; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + swz<D>(16 * np + (lane & 7) + ((lane >> 4) << 3), 2 * kk + ((lane >> 3) & 1)),
                b0, b1, b2, b3);
        mma_bf16_16816(sc[2 * np], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b0, b1);
        mma_bf16_16816(sc[2 * np + 1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b2, b3);
      }
    // online softmax per row; column c of tile nt is context row x + 8 nt + 2 (lane & 3) + e
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float bm = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < kPfRows / 8; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int xc = x + 8 * nt + 2 * (lane & 3) + e;
          const bool ok = xc < n_ctx && xc <= vis[h];
          const float v = ok ? sc[nt][2 * h + e] * scale_log2 : -INFINITY;
          sc[nt][2 * h + e] = v;
          bm = fmaxf(bm, v);
        }
      bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
      bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
      const float mn = fmaxf(mrow[h], bm);
      // a row that has seen nothing yet (mn = -inf) keeps zero weight and scale 1
      const float al = mn == -INFINITY ? 1.0f : exp2f(mrow[h] - mn);
      float ps = 0.0f;
#pragma unroll
      for (int nt = 0; nt < kPfRows / 8; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float pv = mn == -INFINITY ? 0.0f : exp2f(sc[nt][2 * h + e] - mn);
          sc[nt][2 * h + e] = pv;
          ps += pv;
        }
      mrow[h] = mn;
      lrow[h] = lrow[h] * al + ps;
#pragma unroll
      for (int nt = 0; nt < NTD; ++nt) {
        o[nt][2 * h] *= al;
        o[nt][2 * h + 1] *= al;
      }
    }
    // O += P V: P's accumulator pairs are the A fragments of a 16-column k step
#pragma unroll
    for (int kk = 0; kk < kPfRows / 16; ++kk) {
      const uint32_t pa0 = pack_bf16x2(sc[2 * kk][0], sc[2 * kk][1]);
      const uint32_t pa1 = pack_bf16x2(sc[2 * kk][2], sc[2 * kk][3]);
      const uint32_t pa2 = pack_bf16x2(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
      const uint32_t pa3 = pack_bf16x2(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_trans(vb + swz<D>(16 * kk + (lane & 7) + (((lane >> 3) & 1) << 3),
                                  2 * dp + (lane >> 4)),
                      b0, b1, b2, b3);
        mma_bf16_16816(o[2 * dp], pa0, pa1, pa2, pa3, b0, b1);
        mma_bf16_16816(o[2 * dp + 1], pa0, pa1, pa2, pa3, b2, b3);
      }
    }
    __syncthreads();  // every warp is done with stage st before it is refilled
    st ^= 1;
  }

  // row sums over the quad, then O / l for the rows of this call's tokens
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float L = lrow[h];
    L += __shfl_xor_sync(0xffffffffu, L, 1);
    L += __shfl_xor_sync(0xffffffffu, L, 2);
    const int r = (lane >> 2) + 8 * h;
    const int t = t0 + warp * TW + r / G;
    if (t >= T_tok) continue;
    const bool live = len0 + t < cap && L > 0.0f;
    const float inv = live ? 1.0f / L : 0.0f;
    __nv_bfloat16 *orow =
        O + ((static_cast<int64_t>(b) * T_tok + t) * H_q + g * G + r % G) * D + 2 * (lane & 3);
#pragma unroll
    for (int nt = 0; nt < NTD; ++nt)
      *reinterpret_cast<uint32_t *>(orow + 8 * nt) =
          pack_bf16x2(o[nt][2 * h] * inv, o[nt][2 * h + 1] * inv);
  }
}

}  // namespace msa
