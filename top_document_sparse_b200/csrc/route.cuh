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
template <typename T>
__global__ void qnorm_kernel(const T *__restrict__ Qr, int W, int d_r, T *__restrict__ out) {
  const int64_t r = blockIdx.x;
  const int e0 = threadIdx.x * 4;
  const bool active = e0 < W;
  float v[4] = {0.f, 0.f, 0.f, 0.f};
  if (active) load4(Qr + r * W + e0, v);
  float ss = 0.0f;
#pragma unroll
  for (int e = 0; e < 4; ++e) ss = fmaf(v[e], v[e], ss);
  for (int o = d_r / 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.0f / fmaxf(sqrtf(ss), kEps);
#pragma unroll
  for (int e = 0; e < 4; ++e) v[e] *= inv;
  if (active) store4(out + r * W + e0, v);
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
// chunks, then atomic max into state.
__device__ __forceinline__ void epi_doc_max(const float *S, int ldS, int MC, int QB, int64_t b0,
                                            const int *docs, int n_docs, float *state, int tid,
                                            int nthr) {
  for (int p = tid; p < MC * QB; p += nthr) {
    const int q = p / MC, m = p % MC;
    const int d = docs[m];
    if (m > 0 && docs[m - 1] == d) continue;
    float v = S[m * ldS + q];
    for (int m2 = m + 1; m2 < MC && docs[m2] == d; ++m2) v = fmaxf(v, S[m2 * ldS + q]);
    atomic_max_float(state + (b0 + q) * n_docs + d, v);
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
  epi_token_max(S, 33, MC, NR, r0, T_tok, tid, 256);
  __syncthreads();
  const int64_t b0 = r0 / T_tok;
  const int QB = static_cast<int>((r0 + NR - 1) / T_tok - b0 + 1);
  epi_doc_max(S, 33, MC, QB, b0, docs, n_docs, state, tid, 256);
}

// ---------------------------------------------------------------- bf16 path
// Tensor-core route.  A CTA is a persistent loop over (row tile, chunk tile)
// pairs; a chunk tile is 128 chunks, a row tile NT query rows.  Warp 4 is the
// producer: one lane issues TMA loads of 64-feature slices (128 rows x 128 B,
// 128B-swizzled) of the unit router keys into a ring of `stages` buffers, and
// of the normalised query rows (all W features of NT rows, resident while the
// row tile lasts).  Warps 0-3 each own 32 chunks of the tile and run
// mma.sync m16n8k16 (bf16 in, fp32 accumulate) over the slices, then the
// shared epilogue.  Every barrier wait is bounded.
constexpr int kRouteTileC = 128;
constexpr int kRouteSliceBytes = kRouteTileC * 128;  // 16 KiB

template <int NT>
struct RouteLayout {
  static __host__ __device__ size_t q_bytes(int W) { return static_cast<size_t>(W / 64) * NT * 128; }
  static __host__ __device__ size_t s_bytes() { return static_cast<size_t>(kRouteTileC) * (NT + 1) * 4; }
  static __host__ __device__ size_t bytes(int W, int stages) {
    return 1024 /*alignment slack*/ + q_bytes(W) + static_cast<size_t>(stages) * kRouteSliceBytes +
           s_bytes() + kRouteTileC * 4 + (2 * stages + 2) * 8 + 16;
  }
};

template <int NT>
__global__ void __launch_bounds__(160, 1)
route_mma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                 int64_t C, int R, int W, int T_tok, float inv_Hr,
                 const int32_t *__restrict__ chunk_doc, int n_docs, float *__restrict__ state,
                 int n_chunk_tiles, int n_tiles, int stages) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int KS = W / 64;
  uint8_t *Qs = smem;
  uint8_t *Ks = Qs + RouteLayout<NT>::q_bytes(W);
  float *Sb = reinterpret_cast<float *>(Ks + static_cast<size_t>(stages) * kRouteSliceBytes);
  int *docs = reinterpret_cast<int *>(Sb + kRouteTileC * (NT + 1));
  uint64_t *bars = reinterpret_cast<uint64_t *>(docs + kRouteTileC);
  // written only by consumer warps, read only after a consumer barrier, so
  // every consumer warp takes the same abort decision
  volatile int *cons_abort = reinterpret_cast<volatile int *>(bars + 2 * stages + 2);
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + stages);
  const uint32_t qfull = smem_u32(bars + 2 * stages), qempty = smem_u32(bars + 2 * stages + 1);
  const uint32_t qs_addr = smem_u32(Qs), ks_addr = smem_u32(Ks);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  constexpr int LD = NT + 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 4);
    }
    mbar_init(qfull, 1);
    mbar_init(qempty, 4);
    *cons_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 4) {  // ------------------------------------------- producer
    if (lane != 0) return;
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmQ);
    const uint64_t pol = policy_evict_first();
    int it = 0, qloads = 0, cur_rt = -1;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
      const int rt = tile / n_chunk_tiles, ct = tile % n_chunk_tiles;
      if (rt != cur_rt) {
        if (qloads > 0 && !mbar_wait(qempty, (qloads - 1) & 1)) { ok = false; break; }
        mbar_arrive_expect_tx(qfull, static_cast<uint32_t>(KS * NT * 128));
        for (int s = 0; s < KS; ++s) tma_load_2d(qs_addr + s * NT * 128, &tmQ, 64 * s, rt * NT, qfull);
        ++qloads;
        cur_rt = rt;
      }
      for (int s = 0; s < KS; ++s) {
        const int st = it % stages;
        if (it >= stages && !mbar_wait(empty0 + 8 * st, ((it / stages) - 1) & 1)) { ok = false; break; }
        mbar_arrive_expect_tx(full0 + 8 * st, kRouteSliceBytes);
        tma_load_2d_hint(ks_addr + st * kRouteSliceBytes, &tmK, 64 * s, ct * kRouteTileC,
                         full0 + 8 * st, pol);
        ++it;
      }
    }
    if (!ok) {
      raise_device_error(MSA_DEVERR_WAIT_TIMEOUT);
      // let every copy this thread issued land before the CTA can exit
      for (int j = (it > stages ? it - stages : 0); j < it; ++j)
        mbar_wait(full0 + 8 * (j % stages), (j / stages) & 1);
      if (qloads > 0) mbar_wait(qfull, (qloads - 1) & 1);
    }
    return;
  }

  // ----------------------------------------------------------- consumers
  const int tid = threadIdx.x;  // 0..127
  int it = 0, quses = 0, cur_rt = -1;
  bool failed = false;
  for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const int rt = tile / n_chunk_tiles, ct = tile % n_chunk_tiles;
    if (rt != cur_rt) {
      if (quses > 0) {
        __syncwarp();
        if (lane == 0) mbar_arrive(qempty);
      }
      if (!failed && !mbar_wait(qfull, quses & 1)) failed = true;
      ++quses;
      cur_rt = rt;
    }
    float acc[2][NT / 8][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int n = 0; n < NT / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[a][n][e] = 0.0f;

    for (int s = 0; s < KS; ++s, ++it) {
      const int st = it % stages;
      if (!failed && !mbar_wait(full0 + 8 * st, (it / stages) & 1)) failed = true;
      if (!failed) {
        const uint32_t kbase = ks_addr + st * kRouteSliceBytes;
        const uint32_t qbase = qs_addr + s * NT * 128;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t a[2][4];
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            const int row = warp * 32 + mt * 16 + (lane & 15);
            const int chunk = 2 * kk + (lane >> 4);
            ldsm_x4(kbase + row * 128 + ((chunk ^ (row & 7)) << 4), a[mt][0], a[mt][1], a[mt][2],
                    a[mt][3]);
          }
#pragma unroll
          for (int ng = 0; ng < NT / 16; ++ng) {
            const int row = ng * 16 + (lane & 7) + ((lane >> 4) << 3);
            const int chunk = 2 * kk + ((lane >> 3) & 1);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(qbase + row * 128 + ((chunk ^ (row & 7)) << 4), b0, b1, b2, b3);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
              mma_bf16_16816(acc[mt][2 * ng], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b0, b1);
              mma_bf16_16816(acc[mt][2 * ng + 1], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b2, b3);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * st);
    }
    if (failed) *cons_abort = 1;

    // epilogue: scores -> shared, token max, document max -> state
    const int64_t c0 = static_cast<int64_t>(ct) * kRouteTileC;
    const int64_t r0 = static_cast<int64_t>(rt) * NT;
    const int MC = static_cast<int>(C - c0 < kRouteTileC ? C - c0 : kRouteTileC);
    const int NR = static_cast<int>(R - r0 < NT ? R - r0 : NT);
    {
      const int g = lane >> 2, q2 = (lane & 3) * 2;
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int n = 0; n < NT / 8; ++n) {
          const int m = warp * 32 + mt * 16 + g;
          const int col = n * 8 + q2;
          Sb[m * LD + col] = acc[mt][n][0] * inv_Hr;
          Sb[m * LD + col + 1] = acc[mt][n][1] * inv_Hr;
          Sb[(m + 8) * LD + col] = acc[mt][n][2] * inv_Hr;
          Sb[(m + 8) * LD + col + 1] = acc[mt][n][3] * inv_Hr;
        }
    }
    if (tid < MC) docs[tid] = chunk_doc[c0 + tid];
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const bool abort_now = *cons_abort != 0;
    if (!abort_now) epi_token_max(Sb, LD, MC, NR, r0, T_tok, tid, 128);
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const int64_t b0 = r0 / T_tok;
    const int QB = static_cast<int>((r0 + NR - 1) / T_tok - b0 + 1);
    if (!abort_now) epi_doc_max(Sb, LD, MC, QB, b0, docs, n_docs, state, tid, 128);
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (abort_now) break;
  }
  if (failed) raise_device_error(MSA_DEVERR_WAIT_TIMEOUT);
}

}  // namespace msa
