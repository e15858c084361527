// route_tc.cuh -- tensor-core (tcgen05) route score for bf16 memories
// (MSA, b-lab.team summary item 1 "Scalable Sparse Attention"; stage "Online
// Routing & Context Assembly").
//
// s[c, r] = (1/H_r) * <Khat[c], Qhat[r]> over W = H_r * d_r features, with
// Khat the unit router keys (per head) and Qhat the normalised query rows, so
// s is the mean over router heads of the per-head cosines.  A tile is 128
// chunks (UMMA M) x NT query rows (UMMA N); D lives in TMEM.
//
// Warp roles (192 threads):
//   warp 4  one lane: TMA producer -- query rows of the row tile (resident,
//           all W features; or streamed slice by slice, QS) and a ring of
//           64-feature x 128-chunk key slices
//   warp 5  allocates TMEM; one lane issues 4 UMMAs (K = 16 each) per slice
//           and commits them to the slice's "empty" barrier, then commits
//           the finished accumulator to "acc full"
//   warps 0-3  epilogue: while the MMAs run, finds the tile's document runs;
//           then thread t drains TMEM lane t (chunk t of the tile) into
//           registers, scales, takes the max over each document run (warp
//           shuffles; through shared memory after a token max when a query
//           has several rows) and merges into the running state with atomic
//           max reductions
// Two TMEM accumulators alternate, so the epilogue of tile i overlaps the MMAs
// of tile i+1.  Every barrier wait is bounded; a wait that runs out raises
// MSA_DEVERR_WAIT_TIMEOUT, later waits are skipped, in-flight copies and MMAs
// are drained, and TMEM is freed before the CTA exits.
#pragma once
#include "route.cuh"
#include "tc05.cuh"

namespace msa {

// QS (streamed query): the producer copies the row tile's 64-feature query
// slice into each ring stage next to the key slice, instead of keeping all W
// features of the NT query rows resident.  With NT = 64 and W = 1024 the
// resident rows would take 128 KiB and leave room for only four key slices in
// flight; streamed, the ring holds about eight (24 KiB) stages.
template <int NT, bool QS>
struct RouteTcLayout {
  static constexpr int kTileC = 128;
  static constexpr int kSlice = kTileC * 128;  // 16 KiB: 128 rows x 64 bf16
  static constexpr int kQSlice = NT * 128;     // NT rows x 64 bf16
  static constexpr int kStage = kSlice + (QS ? kQSlice : 0);
  static constexpr int kLD = NT + 1;           // epilogue staging row stride (floats)
  static constexpr uint32_t kTmemCols = (2 * NT < 32) ? 32 : 2 * NT;
  static __host__ __device__ size_t q_bytes(int W) {
    return QS ? 0 : static_cast<size_t>(W / 64) * NT * 128;
  }
  static __host__ __device__ size_t bytes(int W, int stages) {
    return 1024 + q_bytes(W) + static_cast<size_t>(stages) * kStage +
           static_cast<size_t>(kTileC) * kLD * 4 + (2 * kTileC + 8) * 4 + (2 * stages + 7) * 8 +
           32;
  }
};

template <int NT, bool QS>
__global__ void __launch_bounds__(192, 1)
route_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                int64_t C, int R, int W, int T_tok, float inv_Hr,
                const int32_t *__restrict__ chunk_doc, int n_docs, float *__restrict__ state,
                int n_chunk_tiles, int n_tiles, int stages) {
  using L = RouteTcLayout<NT, QS>;
  static_assert(NT % 16 == 0 && NT >= 16 && NT <= 128, "UMMA N");
  constexpr bool kRegRuns = NT <= 64;  // document-run max in registers (one-token rows)
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int KS = W / 64;
  uint8_t *Qs = smem;
  uint8_t *Ks = Qs + L::q_bytes(W);
  float *Sb = reinterpret_cast<float *>(Ks + static_cast<size_t>(stages) * L::kStage);
  int *docs = reinterpret_cast<int *>(Sb + L::kTileC * L::kLD);
  int *segs = docs + L::kTileC;  // kTileC + 1 run starts (+ padding)
  uint64_t *bars = reinterpret_cast<uint64_t *>(segs + L::kTileC + 8);
  // bars: full[stages], empty[stages], qfull, qempty, accf[2], acce[2], drain
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * stages + 7);
  volatile int *fail = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + stages);
  const uint32_t qfull = smem_u32(bars + 2 * stages), qempty = smem_u32(bars + 2 * stages + 1);
  const uint32_t accf0 = smem_u32(bars + 2 * stages + 2), acce0 = smem_u32(bars + 2 * stages + 4);
  const uint32_t drain = smem_u32(bars + 2 * stages + 6);
  const uint32_t qs_addr = smem_u32(Qs), ks_addr = smem_u32(Ks);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(qfull, 1);
    mbar_init(qempty, 1);
    mbar_init(accf0, 1);
    mbar_init(accf0 + 8, 1);
    mbar_init(acce0, 128);
    mbar_init(acce0 + 8, 128);
    mbar_init(drain, 1);
    *fail = 0;
    fence_mbar_init();
  }
  if (warp == 5) tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
  tc05_fence_before();
  __syncthreads();
  tc05_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The first tile's first key slices are loaded before the wait for the
  // previous kernel (the query normalisation): router keys are written by no
  // kernel that can still be running here (see qnorm_kernel).  Query slices,
  // documents and state come after the wait.
  int n_pre = 0;
  if (warp == 4 && lane == 0) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmQ);
    if (static_cast<int>(blockIdx.x) < n_tiles) {
      const uint64_t pol = policy_evict_first();
      const int ct0 = static_cast<int>(blockIdx.x) % n_chunk_tiles;
      n_pre = stages < KS ? stages : KS;
      for (int s = 0; s < n_pre; ++s) {
        // with streamed query slices the stage's arrival (and the query bytes) come after the
        // wait, so the phase cannot complete on the keys alone
        if (QS)
          mbar_expect_tx(full0 + 8 * s, L::kSlice);
        else
          mbar_arrive_expect_tx(full0 + 8 * s, L::kStage);
        tma_load_2d_hint(ks_addr + s * L::kStage, &tmK, 64 * s, ct0 * L::kTileC, full0 + 8 * s,
                         pol);
      }
    }
  }
  griddep_wait();  // setup above overlaps the previous kernel's drain
  // The next kernel (the top-k) may be scheduled once every CTA has started the
  // epilogue of its last tile (see the epilogue loop), not earlier: its CTAs
  // only wait for this kernel, and resident early they would hold every SM's
  // spare threads and registers for the whole stream, so that no other work
  // (a fetch on another stream) could run beside it.  With one tile per CTA
  // (the 1M-token decode) that is at once.

  auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
    if (*fail) return false;
    if (mbar_wait(bar, parity)) return true;
    *fail = 1;
    raise_device_error(MSA_DEVERR_WAIT_TIMEOUT);
    return false;
  };

  if (warp == 4) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int it = 0, qloads = 0, cur_rt = -1;
      for (int tile = blockIdx.x; tile < n_tiles && !*fail; tile += gridDim.x) {
        const int rt = tile / n_chunk_tiles, ct = tile % n_chunk_tiles;
        if (!QS && rt != cur_rt) {
          if (qloads > 0 && !wait(qempty, (qloads - 1) & 1)) break;
          mbar_arrive_expect_tx(qfull, static_cast<uint32_t>(KS * NT * 128));
          for (int s = 0; s < KS; ++s)
            tma_load_2d(qs_addr + s * NT * 128, &tmQ, 64 * s, rt * NT, qfull);
          ++qloads;
          cur_rt = rt;
        }
        for (int s = 0; s < KS; ++s) {
          const int st = it % stages;
          if (it >= stages && !wait(empty0 + 8 * st, ((it / stages) - 1) & 1)) break;
          if (it >= n_pre) {
            mbar_arrive_expect_tx(full0 + 8 * st, L::kStage);
            tma_load_2d_hint(ks_addr + st * L::kStage, &tmK, 64 * s, ct * L::kTileC,
                             full0 + 8 * st, pol);
          } else if (QS) {  // key slice already in flight: arrive with the query bytes
            mbar_arrive_expect_tx(full0 + 8 * st, L::kQSlice);
          }
          if (QS)
            tma_load_2d(ks_addr + st * L::kStage + L::kSlice, &tmQ, 64 * s, rt * NT,
                        full0 + 8 * st);
          ++it;
        }
      }
      if (*fail) {  // let every copy issued here land before the CTA can exit
        if (QS)  // stages whose keys went out early but that the loop never reached
          for (int j = it; j < n_pre; ++j) mbar_arrive(full0 + 8 * j);
        const int n_iss = it > n_pre ? it : n_pre;
        for (int j = (n_iss > stages ? n_iss - stages : 0); j < n_iss; ++j)
          mbar_wait(full0 + 8 * (j % stages), (j / stages) & 1);
        if (qloads > 0) mbar_wait(qfull, (qloads - 1) & 1);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16_f32<128, NT>();
      int it = 0, quses = 0, cur_rt = -1, tl = 0;
      bool issued = false;
      for (int tile = blockIdx.x; tile < n_tiles && !*fail; tile += gridDim.x, ++tl) {
        const int rt = tile / n_chunk_tiles;
        if (!QS && rt != cur_rt) {
          if (quses > 0) umma_commit(qempty);  // previous row tile's MMAs are all issued
          if (!wait(qfull, quses & 1)) break;
          ++quses;
          cur_rt = rt;
        }
        const int buf = tl & 1;
        if (tl >= 2 && !wait(acce0 + 8 * buf, ((tl >> 1) - 1) & 1)) break;
        tc05_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(buf * NT);
        bool ok = true;
        for (int s = 0; s < KS; ++s, ++it) {
          const int st = it % stages;
          if (!wait(full0 + 8 * st, (it / stages) & 1)) { ok = false; break; }
          tc05_fence_after();
          const uint32_t a0 = ks_addr + st * L::kStage;
          const uint32_t b0 = QS ? a0 + L::kSlice : qs_addr + s * NT * 128;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(d_tmem, umma_desc_k_sw128(a0 + kk * 32), umma_desc_k_sw128(b0 + kk * 32),
                      idesc, (s | kk) != 0);
          umma_commit(empty0 + 8 * st);
          issued = true;
        }
        if (!ok) break;
        umma_commit(accf0 + 8 * buf);
      }
      if (issued) {  // every MMA has completed before TMEM can be freed
        umma_commit(drain);
        mbar_wait(drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int tid = threadIdx.x;  // 0..127 == TMEM lane == chunk row of the tile
    int tl = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tl) {
      if (tile + static_cast<int>(gridDim.x) >= n_tiles) griddep_launch();  // the last tile
      const int rt = tile / n_chunk_tiles, ct = tile % n_chunk_tiles;
      const int buf = tl & 1;
      const int64_t c0 = static_cast<int64_t>(ct) * L::kTileC;
      const int64_t r0 = static_cast<int64_t>(rt) * NT;
      const int MC = static_cast<int>(C - c0 < L::kTileC ? C - c0 : L::kTileC);
      const int NR = static_cast<int>(R - r0 < NT ? R - r0 : NT);
      // (32-bit: r0 + NR <= R, an int)
      const int r0i = static_cast<int>(r0);
      const int b0 = r0i / T_tok;
      const int QB = (r0i + NR - 1) / T_tok - b0 + 1;
      // the tile's documents and their runs, found while the MMAs run
      if (tid < MC) docs[tid] = chunk_doc[c0 + tid];
      asm volatile("bar.sync 1, 128;" ::: "memory");
      const int n_seg = epi_doc_runs(docs, MC, segs, tid, 128);
      const bool ok = wait(accf0 + 8 * buf, (tl >> 1) & 1);
      const bool okw = __all_sync(0xffffffffu, ok);
      tc05_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16) +
                             static_cast<uint32_t>(buf * NT);
      // After a failed wait the results are void (the error word is set): the
      // writes are skipped (`go`), but every thread still takes every barrier.
      // Shared-memory path: staged 16 columns at a time, token max, run max by columns.
      auto staged = [&]() {
#pragma unroll 4
        for (int c = 0; c < NT; c += 16) {
          float x[16];
          if (okw) tmem_ld16(taddr + c, x);  // (warp-collective: a warp-uniform condition)
#pragma unroll
          for (int i = 0; i < 16; ++i) Sb[tid * L::kLD + c + i] = okw ? x[i] * inv_Hr : 0.0f;
        }
        tc05_fence_before();
        mbar_arrive(acce0 + 8 * buf);  // this accumulator may be overwritten
        const bool go = !*fail;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (go && T_tok > 1) epi_token_max(Sb, L::kLD, MC, NR, r0, T_tok, tid, 128);
        asm volatile("bar.sync 1, 128;" ::: "memory");
        epi_run_max_smem(Sb, L::kLD, QB, segs, n_seg, tid, 128, go);
      };
      if constexpr (kRegRuns) {
        if (T_tok == 1) {  // one token per query: the run max in registers
          float v[NT];
#pragma unroll
          for (int c = 0; c < NT; c += 16) {
            float x[16];
            if (okw) tmem_ld16(taddr + c, x);
#pragma unroll
            for (int i = 0; i < 16; ++i) v[c + i] = okw ? x[i] * inv_Hr : 0.0f;
          }
          tc05_fence_before();
          mbar_arrive(acce0 + 8 * buf);  // this accumulator may be overwritten
          epi_run_max_regs<NT>(v, docs, MC, Sb, L::kLD, tid, 128, !*fail);
        } else {
          staged();
        }
      } else {
        staged();
      }
      const bool go = !*fail;
      if (go) epi_state_merge(Sb, L::kLD, QB, b0, docs, segs, n_seg, n_docs, state, tid, 128);
      asm volatile("bar.sync 1, 128;" ::: "memory");
    }
  }
  tc05_fence_before();
  __syncthreads();
  tc05_fence_after();
  if (warp == 5) tmem_dealloc(tmem, L::kTmemCols);
}

}  // namespace msa
