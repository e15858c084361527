// route.cuh -- online routing score (MSA, b-lab.team summary item 1
// "Scalable Sparse Attention" and stage "Online Routing & Context Assembly"):
//   s[b,t,c] = (1/H_r) sum_h cos(Q_r[b,t,h], Kbar_r[c,h])
//   state[b,d] = max(state[b,d], max_{t, c in d} s[b,t,c])
// Router keys are stored with unit norm per head, so after the query rows are
// normalised (qnorm_kernel) the cosine sum is one dot product of length
// H_r * d_r and the route is a skinny matrix product [C x W] . [W x R] with a
// max epilogue.  The epilogue scales by 1/H_r, reduces over the query's tokens
// and over the document's chunks inside the tile, and max-merges into the
// running state with an atomic float max (exact and order-independent).
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace msa {

// Q_hat[r][h][:] = Q_r[r][h][:] / max(|Q_r[r][h]|, eps).  One CTA per row;
// thread i owns 4 elements; the d_r/4 threads of a head form an aligned group.
// Row r = b * T + t of the output reads input row b * pitch + t.
// The route kernel that follows may start at once: before its own wait it
// only loads router keys, which no kernel of this library that releases its
// dependents early ever writes.  With `early` (the query rows are the
// caller's, which no kernel of this library writes) the rows are normalised
// while the previous kernel still runs, and the wait for it comes last, so
// that this kernel still completes after it; Q_hat was last read by the
// previous route's MMAs, which completed before that route released its
// dependents.
template <typename T>
__global__ void qnorm_kernel(const T *__restrict__ Qr, int W, int d_r, int T_tok, int pitch,
                             T *__restrict__ out, int early) {
  griddep_launch();
  if (!early) griddep_wait();
  const int64_t r = blockIdx.x;
  const int64_t src_row = (r / T_tok) * pitch + r % T_tok;
  const int e0 = threadIdx.x * 4;
  const bool active = e0 < W;
  float v[4] = {0.f, 0.f, 0.f, 0.f};
  if (active) load4(Qr + src_row * W + e0, v);
  float ss = 0.0f;
#pragma unroll
  for (int e = 0; e < 4; ++e) ss = fmaf(v[e], v[e], ss);
  for (int o = d_r / 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.0f / fmaxf(sqrtf(ss), kEps);
#pragma unroll
  for (int e = 0; e < 4; ++e) v[e] *= inv;
  if (active) store4(out + r * W + e0, v);
  if (early) griddep_wait();
}

// ---------------------------------------------------------------- epilogue
// S: scores of chunks c0.. (rows, MC of them) x query rows r0.. (columns).
// Stage 1 (one thread per chunk row): collapse the columns of each query to
// their max, in place, so S[m][q] holds query (r0/T + q)'s max.
__device__ __forceinline__ void epi_token_max(float *S, int ldS, int MC, int NR, int64_t r0,
                                              int T_tok, int tid, int nthr) {
  for (int m = tid; m < MC; m += nthr) {
    float *row = S + m * ldS;
    int64_t b_cur = r0 / T_tok;
    int64_t next_b_row = (b_cur + 1) * T_tok;  // first row of the next query
    float best = row[0];
    int q = 0;
    for (int n = 1; n < NR; ++n) {
      const float v = row[n];
      if (r0 + n >= next_b_row) {
        row[q++] = best;
        best = v;
        next_b_row += T_tok;
      } else {
        best = fmaxf(best, v);
      }
    }
    row[q] = best;
  }
}

// Stage 2: for each (document run inside the tile, query), max over the run's
// chunks, then max-merge into state with an atomic float max.  The atomics
// are reductions (no value comes back), so the merge costs the CTA no memory
// round trip; a max is order-independent, so the result is exact and
// deterministic however the CTAs interleave.  Pieces:
//   epi_doc_runs     run starts of docs[0..MC) -> segs (ordered compaction)
//   epi_run_max_smem run maxima of S by columns (any T)
//   epi_run_max_regs run maxima of register rows by warp shuffles (T == 1)
//   epi_state_merge  S[run start][q] -> state[b0 + q][doc]
constexpr int kEpiMaxWarps = 8;

// All nthr (<= 32 * kEpiMaxWarps) threads must call it (named barrier 2);
// docs[] must be visible to every caller.  Returns the run count; segs[g] is
// the first row of run g and segs[n_seg] = MC.
__device__ __forceinline__ int epi_doc_runs(const int *docs, int MC, int *segs, int tid,
                                            int nthr) {
  const int lane = tid & 31, warp = tid >> 5;
  __shared__ int warp_cnt[kEpiMaxWarps];
  int n_seg = 0;
  for (int base = 0; base < MC; base += nthr) {
    const int m = base + tid;
    const bool start = m < MC && (m == 0 || docs[m] != docs[m - 1]);
    const unsigned bal = __ballot_sync(0xffffffffu, start);
    if (lane == 0) warp_cnt[warp] = __popc(bal);
    asm volatile("bar.sync 2, %0;" ::"r"(nthr) : "memory");
    int before = n_seg;
    for (int w = 0; w < warp; ++w) before += warp_cnt[w];
    if (start) segs[before + __popc(bal & ((1u << lane) - 1))] = m;
    for (int w = 0; w < nthr / 32; ++w) n_seg += warp_cnt[w];
    asm volatile("bar.sync 2, %0;" ::"r"(nthr) : "memory");
  }
  if (tid == 0) segs[n_seg] = MC;
  asm volatile("bar.sync 2, %0;" ::"r"(nthr) : "memory");
  return n_seg;
}

// S[segs[g]][q] = max over run g of column q, in place.  Thread t takes column
// q = t % QB (consecutive lanes, consecutive banks) and every (nthr / QB)-th
// run.  All nthr threads must call it (named barrier 2); `write` may differ
// between threads.
__device__ __forceinline__ void epi_run_max_smem(float *S, int ldS, int QB, const int *segs,
                                                 int n_seg, int tid, int nthr, bool write) {
  const int cols = QB < nthr ? QB : nthr;
  const int per_col = nthr / cols;
  if (write && tid < cols * per_col) {
    const int q0 = tid % cols;
    for (int q = q0; q < QB; q += cols)
      for (int g = tid / cols; g < n_seg; g += per_col) {
        const int m0 = segs[g], m1 = segs[g + 1];
        float x = S[m0 * ldS + q];
        for (int m = m0 + 1; m < m1; ++m) x = fmaxf(x, S[m * ldS + q]);
        S[m0 * ldS + q] = x;
      }
  }
  asm volatile("bar.sync 2, %0;" ::"r"(nthr) : "memory");
}

// Thread tid holds row tid of the tile's scores in v[0..NC).  Leaves, for every
// run, its maxima in the run's first row of S (columns 0..NC).  Inside a warp a
// segmented reduction by shuffles (offsets 1 .. 16: lane l ends up with the max
// over lanes l .. the end of its run in the warp), whatever a run's length; a
// run that goes on into later warps then folds in their lane-0 rows.  All nthr
// threads must call it (named barrier 2); `write` may differ between threads.
template <int NC>
__device__ __forceinline__ void epi_run_max_regs(float (&v)[NC], const int *docs, int MC, float *S,
                                                 int ldS, int tid, int nthr, bool write) {
  const int lane = tid & 31, warp = tid >> 5;
  const int m = tid;
  const int d = m < MC ? docs[m] : -1 - m;  // rows past the tile's chunks: runs of their own
  const bool start = m == 0 || m >= MC || d != docs[m - 1];
  const unsigned starts = __ballot_sync(0xffffffffu, start);
  const unsigned later = lane == 31 ? 0u : starts & (0xffffffffu << (lane + 1));
  const int run_end = later ? __ffs(later) - 1 : 32;  // first lane past my run in this warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const bool take = lane + o < run_end;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const float t = __shfl_down_sync(0xffffffffu, v[c], o);
      v[c] = take ? fmaxf(v[c], t) : v[c];
    }
  }
  if (write && m < MC && (start || lane == 0)) {
#pragma unroll
    for (int c = 0; c < NC; ++c) S[m * ldS + c] = v[c];
  }
  asm volatile("bar.sync 2, %0;" ::"r"(nthr) : "memory");
  if (write && m < MC && start && run_end == 32) {
    for (int j = 32 * (warp + 1); j < MC && docs[j] == d; j += 32)
#pragma unroll
      for (int c = 0; c < NC; ++c) S[m * ldS + c] = fmaxf(S[m * ldS + c], S[j * ldS + c]);
  }
  asm volatile("bar.sync 2, %0;" ::"r"(nthr) : "memory");
}

// state[b0 + q][doc of run g] = max(itself, S[segs[g]][q]) for every (q < QB,
// g < n_seg).  Consecutive threads take consecutive runs -- consecutive
// documents -- of one query, so the reductions coalesce.
__device__ __forceinline__ void epi_state_merge(const float *S, int ldS, int QB, int64_t b0,
                                                const int *docs, const int *segs, int n_seg,
                                                int n_docs, float *state, int tid, int nthr) {
  const int total = n_seg * QB;
  for (int p = tid; p < total; p += nthr) {
    const int q = p / n_seg, g = p - q * n_seg;
    const int m0 = segs[g];
    atomic_max_float(state + (b0 + q) * n_docs + docs[m0], S[m0 * ldS + q]);
  }
}

// ---------------------------------------------------------------- fp32 path
// CUDA-core route for fp32 memories: 32 chunks x 32 query rows per CTA,
// features staged through shared memory 32 at a time (fp32 accumulate).
template <typename T>
__global__ void __launch_bounds__(256)
route_simt_kernel(const T *__restrict__ Khat, const T *__restrict__ Qhat, int64_t C, int R, int W,
                  int T_tok, float inv_Hr, const int32_t *__restrict__ chunk_doc, int n_docs,
                  float *__restrict__ state) {
  __shared__ float Ks[32][33];
  __shared__ float Qs[32][33];
  __shared__ float S[32 * 33];
  __shared__ int docs[32];
  __shared__ int segs[33];
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * 32;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * 32;
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int MC = static_cast<int>(C - c0 < 32 ? C - c0 : 32);
  const int NR = static_cast<int>(R - r0 < 32 ? R - r0 : 32);
  float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
  for (int f0 = 0; f0 < W; f0 += 32) {
    for (int i = tid; i < 1024; i += 256) {
      const int rr = i / 32, ff = i % 32;
      Ks[rr][ff] = rr < MC ? Elem<T>::to_f(Khat[(c0 + rr) * W + f0 + ff]) : 0.0f;
      Qs[rr][ff] = rr < NR ? Elem<T>::to_f(Qhat[(r0 + rr) * W + f0 + ff]) : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int ff = 0; ff < 32; ++ff) {
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 2; ++b) acc[a][b] = fmaf(Ks[ty + 16 * a][ff], Qs[tx + 16 * b][ff], acc[a][b]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < 2; ++b) S[(ty + 16 * a) * 33 + tx + 16 * b] = acc[a][b] * inv_Hr;
  if (tid < MC) docs[tid] = chunk_doc[c0 + tid];
  __syncthreads();
  if (T_tok > 1) epi_token_max(S, 33, MC, NR, r0, T_tok, tid, 256);
  __syncthreads();
  const int64_t b0 = r0 / T_tok;
  const int QB = static_cast<int>((r0 + NR - 1) / T_tok - b0 + 1);
  const int n_seg = epi_doc_runs(docs, MC, segs, tid, 256);
  epi_run_max_smem(S, 33, QB, segs, n_seg, tid, 256, true);
  epi_state_merge(S, 33, QB, b0, docs, segs, n_seg, n_docs, state, tid, 256);
}

// ---------------------------------------------------------------- interleave
// Memory Interleave (Evermind summary sec. 4C, b-lab.team item 3): the
// documents retrieved in a round become part of the next round's query.
// gather_rows_kernel, grid (B): rows[b][0..n_b) = the unit router rows of
// every chunk of ids[b][0..k), in rank order (n_b <= cap); taken[b][id] = 1;
// count[b] = n_b.  pad_rows_kernel then copies row 0 of each query over
// rows[b][n_b..T) so every query has T rows (a repeated row leaves the max
// over rows unchanged).
template <typename T>
__global__ void gather_rows_kernel(const T *__restrict__ keys, const int32_t *__restrict__ ids,
                                   int k, const int64_t *__restrict__ doc_chunk_off, int n_docs,
                                   int W, T *__restrict__ rows, int cap,
                                   uint8_t *__restrict__ taken, int32_t *__restrict__ count) {
  const int b = blockIdx.x;
  __shared__ int s_pos;
  if (threadIdx.x == 0) s_pos = 0;
  __syncthreads();
  for (int r = 0; r < k; ++r) {
    const int d = ids[static_cast<int64_t>(b) * k + r];
    if (d < 0 || d >= n_docs) continue;
    if (threadIdx.x == 0) taken[static_cast<int64_t>(b) * n_docs + d] = 1;
    const int64_t c0 = doc_chunk_off[d], c1 = doc_chunk_off[d + 1];
    const int pos = s_pos;
    const int n = static_cast<int>(min(c1 - c0, static_cast<int64_t>(cap - pos)));
    const int64_t total = static_cast<int64_t>(n) * W / 4;  // 4-element vectors
    T *dst = rows + (static_cast<int64_t>(b) * cap + pos) * W;
    const T *src = keys + c0 * W;
    for (int64_t i = threadIdx.x; i < total; i += blockDim.x) {
      float v[4];
      load4(src + 4 * i, v);
      store4(dst + 4 * i, v);
    }
    __syncthreads();
    if (threadIdx.x == 0) s_pos = pos + n;
    __syncthreads();
  }
  if (threadIdx.x == 0) count[b] = s_pos;
}

template <typename T>
__global__ void pad_rows_kernel(T *__restrict__ rows, int cap, int W,
                                const int32_t *__restrict__ count, int T_rows) {
  const int b = blockIdx.x;
  const int n = count[b];
  if (n <= 0) {  // no new rows: zero rows (their state row is saved and restored around the route)
    const int64_t total = static_cast<int64_t>(T_rows) * W;
    for (int64_t i = threadIdx.x; i < total; i += blockDim.x)
      rows[static_cast<int64_t>(b) * cap * W + i] = Elem<T>::from_f(0.0f);
    return;
  }
  if (n >= T_rows) return;
  const T *src = rows + static_cast<int64_t>(b) * cap * W;
  const int64_t per = W / 4;
  const int64_t total = static_cast<int64_t>(T_rows - n) * per;
  for (int64_t i = threadIdx.x; i < total; i += blockDim.x) {
    const int64_t row = n + i / per, e = (i % per) * 4;
    float v[4];
    load4(src + e, v);
    store4(rows + (static_cast<int64_t>(b) * cap + row) * W + e, v);
  }
}

// grid (B): for the queries with no new rows this round (count[b] == 0), copy
// state row b to saved (dir 0, before the route) or back (dir 1, after it), so
// that routing their padding rows leaves their running state as it was.
__global__ void hold_state_kernel(float *__restrict__ state, float *__restrict__ saved,
                                  const int32_t *__restrict__ count, int n_docs, int dir) {
  const int b = blockIdx.x;
  if (count[b] != 0) return;
  float *st = state + static_cast<int64_t>(b) * n_docs;
  float *sv = saved + static_cast<int64_t>(b) * n_docs;
  for (int d = threadIdx.x; d < n_docs; d += blockDim.x) {
    if (dir == 0)
      sv[d] = st[d];
    else
      st[d] = sv[d];
  }
}

// Adaptive Memory Interleave, after round r's top-k (one thread per query): a
// query still active whose best new document scores below stop_score stops
// (active[b] = 0); a stopped query's ids / scores of this round become -1 /
// -inf (nothing of the round enters its context); an active one records
// n_rounds[b] = r + 1.
__global__ void interleave_stop_kernel(int32_t *__restrict__ ids, float *__restrict__ scores,
                                       int B, int k, float stop_score,
                                       uint8_t *__restrict__ active, int32_t *__restrict__ n_rounds,
                                       int round) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  int32_t *id = ids + static_cast<int64_t>(b) * k;
  float *sc = scores + static_cast<int64_t>(b) * k;
  if (active[b] && !(sc[0] >= stop_score)) active[b] = 0;  // (a -inf best score stops too)
  if (active[b]) {
    n_rounds[b] = round + 1;
    return;
  }
  for (int r = 0; r < k; ++r) {
    id[r] = -1;
    sc[r] = -INFINITY;
  }
}

}  // namespace msa
