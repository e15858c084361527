// prefill_tc.cuh -- multi-token (prefill) sparse GQA attention on the
// 5th-generation tensor cores (MSA, b-lab.team summary item 1 "Scalable Sparse
// Attention" and "Global RoPE", stage "Sparse Generation"): the call's tokens
// attend over [pooled K/V of the retrieved documents' chunks, all visible] ++
// [local cache rows, causal: token t sees local rows up to cache_len + t],
// with Q rotated at pos_offset + cache_len + t.
//
// One CTA per (query, kv head, pair of adjacent tiles of 128 query rows); a
// row is a (token, query head of the GQA group) pair, so a tile holds 128 / G
// tokens.  Both tiles share every K/V block the CTA loads.  The context
// streams through in blocks of 64 rows, the local cache blocks first (their
// rows need no chunk table, so the first loads start at once), then the
// retrieved chunks; the online softmax does not depend on the order.  Per tile
// and block:
//   S   = Q K^T           tcgen05.mma, M = 128 query rows, N = 64 context
//                          rows, K = D; Q and the K block in shared memory
//                          (K-major, 128-byte swizzle); S in one of two TMEM
//                          buffers, so Q K^T of a later block runs while the
//                          softmax works on this one
//   P   = exp2(S - m)     the tile's four softmax warps: warp w reads TMEM
//                          lanes 32 (w % 4) .. (thread = query row), masks the
//                          diagonal and ragged blocks, keeps the row's
//                          reference max m and sum l, writes P as bf16 to the
//                          tile's P buffer and, when the row's max rises more
//                          than 8 (log2 units) above m, moves m and rescales
//                          its row of O in TMEM; below that P stays under 2^8
//                          and the result is the same
//   O  += P V             tcgen05.mma, M = 128, N = D, K = 64 context rows; V
//                          read MN-major straight from its row-major block
// Roles (warp-specialised, synchronised by mbarriers only):
//   warps 0-3, 4-7  tile A, tile B: rotate the Q tile into shared memory, the
//                   softmax, then O / l to global memory
//   warp 8          owns TMEM (all 512 columns: S buffers and O of both
//                   tiles); lane 0 issues every MMA as soon as its inputs are
//                   ready, in whatever order they become ready
//   warps 9-10      stream K/V blocks through a ring of NS stages:
//                   whole local blocks by TMA (one thread), the ragged last
//                   local block and the retrieved chunks (through the chunk
//                   table, which warp 9 builds after the first local blocks are
//                   in flight) by cp.async, each lane's copies arriving on the
//                   stage's barrier when they complete; a stage is refilled once
//                   every P V that reads it has completed.  The softmax and the
//                   MMA issuer take the local blocks before they wait for the
//                   table.
// Every wait is bounded: on timeout the CTA raises MSA_DEVERR_WAIT_TIMEOUT,
// every role skips the rest (the outputs are then void), and issued MMAs are
// drained before TMEM is freed.
#pragma once
#include "attend.cuh"
#include "tc05.cuh"

namespace msa {

constexpr int kPtcRows = 128;             // query rows per tile (UMMA M)
constexpr int kPtcBlk = 64;               // context rows per block (UMMA N of S, K of P V)
constexpr int kPtcMaxStages = 4;          // largest K/V ring depth the barriers provide for
constexpr int kPtcLoadWarps = 2;          // warps 9 .. 9 + kPtcLoadWarps - 1 stream K/V
constexpr int kPtcThreads = 32 * (9 + kPtcLoadWarps);
constexpr uint32_t kPtcTmemCols = 512;
// TMEM columns: S of tile x at 128 x + 64 (u % 2) (u = the tile's block count), O of tile x
// at 256 + 128 x
constexpr uint32_t kPtcTmemO = 256;

// mbarriers of the prefill kernel
enum {
  kPbFull0 = 0,                      // stage s holds its block (the copies of every loader lane)
  kPbEmpty0 = kPtcMaxStages,         // every P V reading stage s has completed (commit)
  kPbS0 = 2 * kPtcMaxStages,         // S buffer (tile x, u % 2) is computed (commit) [4]
  kPbQ0 = kPbS0 + 4,              // tile x's rotated Q is in shared memory (128 threads) [2]
  kPbP0 = kPbQ0 + 2,              // tile x's P is written and O rescaled (128 threads) [2]
  kPbO0 = kPbP0 + 2,              // tile x's P V has completed (commit) [2]
  kPbTab = kPbO0 + 2,             // the chunk table and n_mem are ready (loader lane 0)
  kPbDrain = kPbTab + 1,          // every MMA has completed (commit)
  kPbN = 24
};
static_assert(kPbDrain < kPbN, "barrier slots");

template <int D, int NS>
struct PtcSmem {
  static_assert(NS >= 2 && NS <= kPtcMaxStages, "ring depth");
  static constexpr int kPanels = D / 64;
  static constexpr int kQBytes = kPanels * kPtcRows * 128;   // [panel][128 rows][128 B]
  static constexpr int kKVBytes = kPanels * kPtcBlk * 128;   // [panel][64 rows][128 B]
  static constexpr int kPBytes = kPtcRows * 128;             // [128 rows][64 ctx x 2 B]
  static constexpr int kStage = 2 * kKVBytes;                // K then V
  // Q (2 tiles) | P (2 tiles) | stages | barriers | TMEM slot, fail, n_mem | prefix + bases | table
  static constexpr int kFixed = 1024 + 2 * kQBytes + 2 * kPBytes + NS * kStage + kPbN * 8 +
                                16 + (2 * kMaxTopK + 1) * 4;
  static int bytes(int table_cap) { return kFixed + table_cap * 4; }
};

// Byte offset of 16-byte chunk c (0 .. D/8) of row r of a [panel][rows][128 B]
// tile of `rows` rows (128-byte swizzle: chunk index XOR row % 8).
__device__ __forceinline__ uint32_t ptc_swz(int r, int c, int rows) {
  return static_cast<uint32_t>((c >> 3) * (rows * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// The chunk table of query b built by one warp (the loader): table[x] = chunk
// row of context row x < n_mem, ranks in order; the same rows as
// build_chunk_table.  Returns n_mem in every lane.
__device__ __forceinline__ int build_chunk_table_warp(const int32_t *__restrict__ ids_b, int k,
                                                      const int64_t *__restrict__ doc_chunk_off,
                                                      int n_docs, const int32_t *__restrict__ slots_b,
                                                      int slot_chunks, int *table, int *pre,
                                                      int *base, int table_cap, int lane) {
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
    // (a rank that would overflow the table contributes nothing; host validation keeps
    // k * max_doc_chunks <= table_cap)
    if (r < k) pre[r] = excl + cnt[h] > table_cap ? min(excl, table_cap) : excl;
    run += __shfl_sync(0xffffffffu, v, 31);
  }
  const int n_mem = min(run, table_cap);
  if (lane == 0) pre[k] = n_mem;
  __syncwarp();
  for (int x = lane; x < n_mem; x += 32) {
    int lo = 0, hi = k - 1;  // last rank r with pre[r] <= x
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pre[mid] <= x) lo = mid; else hi = mid - 1;
    }
    table[x] = base[lo] + (x - pre[lo]);
  }
  __syncwarp();
  return n_mem;
}

// grid n_pairs * B * H_kv (n_pairs = ceil(ceil(T * G / 128) / 2)), block
// kPtcThreads, one CTA per SM: the tile pairs of one (query, kv head) are
// adjacent in launch order, so they run at about the same time and read the
// shared context from L2, the pair with the most context first.  append_kernel has written the call's rows to the cache before this
// kernel runs.  tm_k / tm_v map the local cache as [B * cap rows][H_kv][D]
// with box {64 of D, 1 head, 64 rows} (128-byte swizzle): a whole local block
// of the CTA's kv head is two TMA loads per tensor.
template <int D, int G, int NS>
__global__ void __launch_bounds__(kPtcThreads, 1)
attend_prefill_tc_kernel(const __nv_bfloat16 *__restrict__ content,
                         const int32_t *__restrict__ ids, int k,
                         const int64_t *__restrict__ doc_chunk_off, int n_docs,
                         const int32_t *__restrict__ slots, int slot_chunks, int H_kv,
                         const __nv_bfloat16 *__restrict__ Q, int T_tok,
                         const __nv_bfloat16 *__restrict__ K_cache,
                         const __nv_bfloat16 *__restrict__ V_cache,
                         const int32_t *__restrict__ cache_len, int cap, int pos_offset,
                         const float2 *__restrict__ rope, float scale_log2, int table_cap,
                         __nv_bfloat16 *__restrict__ O, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, int n_pairs) {
  static_assert(D == 128, "the tensor-core prefill takes head_dim 128");
  static_assert(G >= 1 && G <= 16 && kPtcRows % G == 0, "GQA group");
  using Sm = PtcSmem<D, NS>;
  constexpr int TT = kPtcRows / G;  // tokens per tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *qs0 = sm;                                   // Q of tile x at qs0 + x * kQBytes
  uint8_t *ps0 = qs0 + 2 * Sm::kQBytes;                // P of tile x at ps0 + x * kPBytes
  uint8_t *stage0 = ps0 + 2 * Sm::kPBytes;             // stage s at stage0 + s * kStage
  uint64_t *bars = reinterpret_cast<uint64_t *>(stage0 + NS * Sm::kStage);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kPbN);
  volatile int *fail = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *n_mem_s = reinterpret_cast<volatile int *>(tmem_slot + 2);
  int *pre = reinterpret_cast<int *>(tmem_slot + 4);
  int *base = pre + (kMaxTopK + 1);
  int *table = base + kMaxTopK;
  auto bar = [&](int i) { return smem_u32(bars + i); };

  const int H_q = H_kv * G;
  const int bg = static_cast<int>(blockIdx.x / n_pairs);
  const int b = bg / H_kv, g = bg % H_kv;
  const int pair = n_pairs - 1 - static_cast<int>(blockIdx.x % n_pairs);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t kv = static_cast<int64_t>(H_kv) * D;
  const int half = D / 2;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(bar(kPbFull0 + i), 32 * kPtcLoadWarps);
      mbar_init(bar(kPbEmpty0 + i), 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(bar(kPbS0 + i), 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(kPbQ0 + x), 128);
      mbar_init(bar(kPbP0 + x), 128);
      mbar_init(bar(kPbO0 + x), 1);
    }
    mbar_init(bar(kPbTab), 1);
    mbar_init(bar(kPbDrain), 1);
    *fail = 0;
    fence_mbar_init();
  }
  if (warp == 8) tmem_alloc(smem_u32(tmem_slot), kPtcTmemCols);
  if (warp == 9 && lane == 0) {
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  griddep_wait();
  griddep_launch();
  const int len0 = cache_len[b];
  tc05_fence_before();
  __syncthreads();  // barriers, the fail flag and the TMEM address are visible
  tc05_fence_after();
  const uint32_t tmem = *tmem_slot;

  // the two tiles: tokens [t0x, t0x + TT), their local rows [0, n_loc[x]), nbl[x] local blocks
  int t0[2], n_loc[2], nbl[2];
  bool act[2];
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    t0[x] = (2 * pair + x) * TT;
    act[x] = t0[x] < T_tok;
    const int t_last = min(t0[x] + TT, T_tok) - 1;
    n_loc[x] = act[x] ? max(0, min(len0 + t_last + 1, cap)) : 0;
    nbl[x] = (n_loc[x] + kPtcBlk - 1) / kPtcBlk;
  }
  // block j < nbL: local rows [64 j, 64 j + 64); block j >= nbL: chunk rows [64 (j - nbL), ...)
  const int nbL = max(nbl[0], nbl[1]);
  const int n_loc_max = max(n_loc[0], n_loc[1]);
  // does tile x read block j (every tile reads every memory block)
  auto uses = [&](int x, int j) { return act[x] && (j < nbl[x] || j >= nbL); };
  // the u-th block tile x reads
  auto blk_of = [&](int x, int u) { return u < nbl[x] ? u : u + (nbL - nbl[x]); };

  // bounded wait; false (and every later wait false at once) after a timeout anywhere
  auto wait = [&](int i, uint32_t parity) -> bool {
    if (*fail) return false;
    if (mbar_wait(bar(i), parity)) return true;
    *fail = 1;
    raise_device_error(MSA_DEVERR_WAIT_TIMEOUT);
    return false;
  };

  if (warp >= 9) {
    // ------------------------------------------------------------ loaders
    const int lw = warp - 9;
    // lane: 16-byte chunk lane % 16 of rows (lane / 16) + 2 lw, then every 2 kPtcLoadWarps
    const int c = lane & 15, r0 = (lane >> 4) + 2 * lw;
    int n_mem = 0;
    auto issue = [&](int j) {
      uint8_t *kb = stage0 + (j % NS) * Sm::kStage;
      uint8_t *vb = kb + Sm::kKVBytes;
#pragma unroll 4
      for (int r = r0; r < kPtcBlk; r += 2 * kPtcLoadWarps) {
        const __nv_bfloat16 *ksrc = K_cache, *vsrc = V_cache;
        bool ok;
        if (j < nbL) {
          const int l = j * kPtcBlk + r;
          ok = l < n_loc_max;
          const int64_t row = (static_cast<int64_t>(b) * cap + l) * kv + g * D;
          if (ok) {
            ksrc = K_cache + row;
            vsrc = V_cache + row;
          }
        } else {
          const int x = (j - nbL) * kPtcBlk + r;
          ok = x < n_mem;
          if (ok) {
            ksrc = content + static_cast<int64_t>(table[x]) * 2 * kv + g * D;
            vsrc = ksrc + kv;
          }
        }
        cp_async_16(smem_u32(kb + ptc_swz(r, c, kPtcBlk)), ksrc + c * 8, ok);
        cp_async_16(smem_u32(vb + ptc_swz(r, c, kPtcBlk)), vsrc + c * 8, ok);
      }
      cp_async_commit();
    };
    // block j into stage j % NS: a whole local block by TMA (every other loader lane arrives
    // at once), otherwise each lane's copies arrive on the stage's barrier once they land
    auto issue_arrive = [&](int j) {
      const uint32_t fb = bar(kPbFull0 + j % NS);
      if (j < nbL && (j + 1) * kPtcBlk <= n_loc_max) {
        if (lw == 0 && lane == 0) {
          mbar_arrive_expect_tx(fb, static_cast<uint32_t>(Sm::kStage));
          const uint32_t kb = smem_u32(stage0 + (j % NS) * Sm::kStage);
          const int row = b * cap + j * kPtcBlk;
          const uint64_t keep = policy_evict_last();  // the other tiles of (b, g) read it too
#pragma unroll
          for (int p = 0; p < Sm::kPanels; ++p) {
            tma_load_3d_hint(kb + p * (kPtcBlk * 128), &tm_k, 64 * p, g, row, fb, keep);
            tma_load_3d_hint(kb + Sm::kKVBytes + p * (kPtcBlk * 128), &tm_v, 64 * p, g, row, fb,
                             keep);
          }
        } else {
          mbar_arrive(fb);
        }
      } else {
        issue(j);
        cp_async_mbar_arrive_noinc(fb);
      }
    };
    // the first local blocks go out before the chunk table is built
    int issued = 0;
    while (issued < min(NS, nbL)) issue_arrive(issued++);
    if (lw == 0) {
      n_mem = build_chunk_table_warp(ids + static_cast<int64_t>(b) * k, k, doc_chunk_off, n_docs,
                                     slots ? slots + static_cast<int64_t>(b) * k : nullptr,
                                     slot_chunks, table, pre, base, table_cap, lane);
      if (lane == 0) {
        *n_mem_s = n_mem;
        mbar_arrive(bar(kPbTab));
      }
    } else {
      n_mem = __all_sync(0xffffffffu, wait(kPbTab, 0)) ? *n_mem_s : 0;
    }
    const int nblk = *fail ? 0 : nbL + (n_mem + kPtcBlk - 1) / kPtcBlk;
    while (issued < min(NS, nblk)) issue_arrive(issued++);
    // block j >= NS refills stage j % NS once every P V reading block j - NS has completed
    for (; issued < nblk; ++issued) {
      if (!wait(kPbEmpty0 + issued % NS, ((issued - NS) / NS) & 1)) break;
      issue_arrive(issued);
    }
    cp_async_wait<0>();
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // until the chunk table is known, only the local blocks
      int n_u[2] = {act[0] ? nbl[0] : 0, act[1] ? nbl[1] : 0};
      bool have_tab = false;
      constexpr uint32_t idesc_s = umma_idesc_bf16_f32<kPtcRows, kPtcBlk>();
      constexpr uint32_t idesc_o = umma_idesc_bf16_f32_bmn<kPtcRows, D>();
      bool ok = true;
#pragma unroll
      for (int x = 0; x < 2; ++x)
        if (act[x]) ok = ok && wait(kPbQ0 + x, 0);
      int next_s[2] = {0, 0}, next_pv[2] = {0, 0};
      uint32_t one_done = 0;  // bit s: one of the two P V reading stage s's block was issued
      long long t_prog = clock64();
      while (ok && (!have_tab || next_pv[0] < n_u[0] || next_pv[1] < n_u[1])) {
        bool prog = false;
        if (!have_tab && mbar_test_wait(bar(kPbTab), 0)) {
          have_tab = true;
          const int nbm = (*n_mem_s + kPtcBlk - 1) / kPtcBlk;
#pragma unroll
          for (int x = 0; x < 2; ++x) n_u[x] = act[x] ? nbl[x] + nbm : 0;
          prog = true;
        }
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          // P V of the tile's block next_pv as soon as its P is written (and O rescaled)
          if (next_pv[x] < n_u[x] && mbar_test_wait(bar(kPbP0 + x), next_pv[x] & 1)) {
            tc05_fence_after();
            const int j = blk_of(x, next_pv[x]);
            const uint32_t p_addr = smem_u32(ps0 + x * Sm::kPBytes);
            const uint32_t v_addr = smem_u32(stage0 + (j % NS) * Sm::kStage) + Sm::kKVBytes;
#pragma unroll
            for (int ks = 0; ks < kPtcBlk / 16; ++ks)
              umma_bf16(tmem + kPtcTmemO + 128 * x, umma_desc_k_sw128(p_addr + ks * 32),
                        umma_desc_mn_sw128(v_addr + ks * 16 * 128, Sm::kKVBytes / Sm::kPanels),
                        idesc_o, (next_pv[x] | ks) != 0);
            umma_commit(bar(kPbO0 + x));
            const uint32_t bit = 1u << (j % NS);
            if (!(uses(0, j) && uses(1, j)) || (one_done & bit)) {  // the last P V reading j
              one_done &= ~bit;
              umma_commit(bar(kPbEmpty0 + j % NS));
            } else {
              one_done |= bit;
            }
            ++next_pv[x];
            prog = true;
          }
          // Q K^T of the tile's block next_s once it has landed and its S buffer is free (the
          // softmax has read the S two blocks back: its P is written)
          if (next_s[x] < n_u[x] && next_s[x] - 2 < next_pv[x]) {
            const int j = blk_of(x, next_s[x]);
            if (mbar_test_wait(bar(kPbFull0 + j % NS), (j / NS) & 1)) {
              // the loaders' cp.async writes (generic proxy) before the tensor cores read them
              fence_proxy_async_smem();
              tc05_fence_after();
              const uint32_t q_addr = smem_u32(qs0 + x * Sm::kQBytes);
              const uint32_t k_addr = smem_u32(stage0 + (j % NS) * Sm::kStage);
              const uint32_t d_s = tmem + 128 * x + kPtcBlk * (next_s[x] & 1);
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t pa = static_cast<uint32_t>((kk >> 2) * kPtcRows * 128 + (kk & 3) * 32);
                const uint32_t pb = static_cast<uint32_t>((kk >> 2) * kPtcBlk * 128 + (kk & 3) * 32);
                umma_bf16(d_s, umma_desc_k_sw128(q_addr + pa), umma_desc_k_sw128(k_addr + pb),
                          idesc_s, kk != 0);
              }
              umma_commit(bar(kPbS0 + 2 * x + (next_s[x] & 1)));
              ++next_s[x];
              prog = true;
            }
          }
        }
        if (prog) {
          t_prog = clock64();
        } else if (*fail) {
          ok = false;
        } else if (clock64() - t_prog > kWaitBudgetCycles) {
          *fail = 1;
          raise_device_error(MSA_DEVERR_WAIT_TIMEOUT);
          ok = false;
        }
      }
      // every MMA issued here completes before TMEM is freed
      umma_commit(bar(kPbDrain));
      mbar_wait(bar(kPbDrain), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax, tile x
    const int x = warp >> 2;
    const int tid = threadIdx.x & 127;
    uint8_t *qs = qs0 + x * Sm::kQBytes;
    uint8_t *psm = ps0 + x * Sm::kPBytes;
    const int tq0 = x ? t0[1] : t0[0];
    const int nbl_x = x ? nbl[1] : nbl[0];
    const int n_loc_x = x ? n_loc[1] : n_loc[0];
    const bool act_x = x ? act[1] : act[0];
    // the tile's rotated query rows (row r = token tq0 + r / G, head g * G + r % G), in
    // 16-byte pieces: item (token, chunk c of the lower half) rotates elements [8c, 8c + 8)
    // with [half + 8c, half + 8c + 8) of the token's G heads, one RoPE load for all of them,
    // every load of a batch of heads issued before its stores.  Rows past the call's tokens
    // or the cache are zero.
    {
      constexpr int HC = D / 16;         // 16-byte chunks in half a row
      constexpr int GB = G < 4 ? G : 4;  // heads per batch of loads
      const uint64_t stream = policy_evict_first();  // Q is read once: keep the cache in L2
      for (int it = tid; it < TT * HC; it += 128) {
        const int tt = it / HC, c = it % HC, t = tq0 + tt;
        const bool live = t < T_tok && len0 + t < cap;
        float2 cs[8];
        const __nv_bfloat16 *q0 = Q;
        if (live) {
          const float4 *cp = reinterpret_cast<const float4 *>(
              rope + static_cast<int64_t>(pos_offset + len0 + t) * half + c * 8);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float4 v = __ldg(cp + u);
            cs[2 * u] = make_float2(v.x, v.y);
            cs[2 * u + 1] = make_float2(v.z, v.w);
          }
          q0 = Q + ((static_cast<int64_t>(b) * T_tok + t) * H_q + g * G) * D + c * 8;
        }
#pragma unroll
        for (int h0 = 0; h0 < G; h0 += GB) {
          uint4 lo[GB], hi[GB];
#pragma unroll
          for (int h = 0; h < GB; ++h) {
            lo[h] = live ? ld_nc_v4_hint(q0 + (h0 + h) * D, stream) : make_uint4(0, 0, 0, 0);
            hi[h] = live ? ld_nc_v4_hint(q0 + (h0 + h) * D + half, stream) : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int h = 0; h < GB; ++h) {
            const int r = tt * G + h0 + h;
            const __nv_bfloat162 *a = reinterpret_cast<const __nv_bfloat162 *>(&lo[h]);
            const __nv_bfloat162 *e = reinterpret_cast<const __nv_bfloat162 *>(&hi[h]);
            uint32_t wl[4], wh[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const float2 fa = __bfloat1622float2(a[p]), fe = __bfloat1622float2(e[p]);
              const float2 c0 = live ? cs[2 * p] : make_float2(0.0f, 0.0f);
              const float2 c1 = live ? cs[2 * p + 1] : make_float2(0.0f, 0.0f);
              wl[p] = pack_bf16x2(fa.x * c0.x - fe.x * c0.y, fa.y * c1.x - fe.y * c1.y);
              wh[p] = pack_bf16x2(fe.x * c0.x + fa.x * c0.y, fe.y * c1.x + fa.y * c1.y);
            }
            *reinterpret_cast<uint4 *>(qs + ptc_swz(r, c, kPtcRows)) =
                make_uint4(wl[0], wl[1], wl[2], wl[3]);
            *reinterpret_cast<uint4 *>(qs + ptc_swz(r, c + HC, kPtcRows)) =
                make_uint4(wh[0], wh[1], wh[2], wh[3]);
          }
        }
      }
    }
    fence_proxy_async_smem();  // Q becomes visible to the tensor cores
    mbar_arrive(bar(kPbQ0 + x));

    const int r = tid;  // the row = the TMEM lane
    const int t_row = tq0 + r / G;
    // the local blocks first; the chunk table (n_mem) only when they are done
    int n_u = act_x ? nbl_x : 0, n_mem = 0;
    bool have_tab = false;
    const int vis_loc = min(len0 + t_row, n_loc_x - 1);  // last visible local row of the row
    float m_run = -INFINITY, l_run = 0.0f;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tmem_o = tmem + kPtcTmemO + 128 * x;
    bool okw = true;
    for (int u = 0;; ++u) {
      if (u >= n_u && !have_tab) {
        have_tab = true;
        okw = __all_sync(0xffffffffu, wait(kPbTab, 0));
        if (!okw) break;
        n_mem = *n_mem_s;
        n_u = act_x ? nbl_x + (n_mem + kPtcBlk - 1) / kPtcBlk : 0;
      }
      if (u >= n_u) break;
      okw = __all_sync(0xffffffffu, wait(kPbS0 + 2 * x + (u & 1), (u >> 1) & 1));
      if (!okw) break;
      tc05_fence_after();
      // the row's last visible column of this block
      const int lim = u < nbl_x ? vis_loc - u * kPtcBlk : n_mem - 1 - (u - nbl_x) * kPtcBlk;
      float s[kPtcBlk];
      static_assert(kPtcBlk == 64, "one 64-column TMEM load per block");
      tmem_ld64(tmem + 128 * x + kPtcBlk * (u & 1) + lane_base, s);
      if (lim < kPtcBlk - 1) {  // a diagonal or ragged block: mask
#pragma unroll
        for (int i = 0; i < kPtcBlk; ++i) s[i] = i <= lim ? s[i] : -INFINITY;
      }
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int i = 0; i < kPtcBlk; ++i) mx[i & 3] = fmaxf(mx[i & 3], s[i]);
      // block max in log2 units (scale_log2 > 0)
      const float bm = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * scale_log2;
      // the reference max moves only when the block's max exceeds it by more than 8
      const float m_new = (m_run == -INFINITY || bm > m_run + 8.0f) ? fmaxf(m_run, bm) : m_run;
      const float alpha = m_new == m_run ? 1.0f : ex2_approx(m_run - m_new);
      const float mo = m_new == -INFINITY ? 0.0f : m_new;  // masked entries give 2^-inf = 0
      float ps[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int i = 0; i < kPtcBlk; ++i) {
        s[i] = ex2_approx(fmaf(s[i], scale_log2, -mo));
        ps[i & 3] += s[i];
      }
      l_run = l_run * alpha + (ps[0] + ps[1]) + (ps[2] + ps[3]);
      m_run = m_new;
      if (u > 0) {
        // the tile's previous P V has completed (waited at every block, so the barrier's
        // phases are never ambiguous): the P buffer is free, and O's row is rescaled when
        // the max rose.  TMEM loads and stores are warp-collective: the warp takes them
        // when any of its rows needs it, each thread with its own factor.
        okw = __all_sync(0xffffffffu, wait(kPbO0 + x, (u - 1) & 1));
        if (!okw) break;
        tc05_fence_after();
        if (__any_sync(0xffffffffu, alpha < 1.0f)) {
#pragma unroll 1
          for (int cc = 0; cc < D; cc += 16) {
            float o[16];
            tmem_ld16(tmem_o + lane_base + cc, o);
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] *= alpha;
            tmem_st16(tmem_o + lane_base + cc, o);
          }
        }
      }
#pragma unroll
      for (int cc = 0; cc < kPtcBlk; cc += 8) {
        uint4 w;
        w.x = pack_bf16x2(s[cc], s[cc + 1]);
        w.y = pack_bf16x2(s[cc + 2], s[cc + 3]);
        w.z = pack_bf16x2(s[cc + 4], s[cc + 5]);
        w.w = pack_bf16x2(s[cc + 6], s[cc + 7]);
        *reinterpret_cast<uint4 *>(psm + ptc_swz(r, cc / 8, kPtcRows)) = w;
      }
      fence_proxy_async_smem();  // P becomes visible to the tensor cores
      tc05_fence_before();
      mbar_arrive(bar(kPbP0 + x));
    }
    // O / l for the rows of this call's tokens (TMEM loads by whole warps)
    const bool row_out = act_x && t_row < min(tq0 + TT, T_tok);
    if (okw && n_u > 0) okw = __all_sync(0xffffffffu, wait(kPbO0 + x, (n_u - 1) & 1));
    __nv_bfloat16 *orow = O + ((static_cast<int64_t>(b) * T_tok + t_row) * H_q + g * G + r % G) * D;
    if (okw && n_u > 0) {
      tc05_fence_after();
      const bool live = len0 + t_row < cap && l_run > 0.0f;
      const float inv = live ? 1.0f / l_run : 0.0f;
      const uint64_t stream = policy_evict_first();  // O is not read here again
#pragma unroll 1
      for (int cc = 0; cc < D; cc += 16) {
        float o[16];
        tmem_ld16(tmem_o + lane_base + cc, o);
        if (!row_out) continue;
        uint4 w0, w1;
        w0.x = pack_bf16x2(o[0] * inv, o[1] * inv);
        w0.y = pack_bf16x2(o[2] * inv, o[3] * inv);
        w0.z = pack_bf16x2(o[4] * inv, o[5] * inv);
        w0.w = pack_bf16x2(o[6] * inv, o[7] * inv);
        w1.x = pack_bf16x2(o[8] * inv, o[9] * inv);
        w1.y = pack_bf16x2(o[10] * inv, o[11] * inv);
        w1.z = pack_bf16x2(o[12] * inv, o[13] * inv);
        w1.w = pack_bf16x2(o[14] * inv, o[15] * inv);
        st_v4_hint(orow + cc, w0, stream);
        st_v4_hint(orow + cc + 8, w1, stream);
      }
    } else if (row_out) {
      for (int cc = 0; cc < D; cc += 8) *reinterpret_cast<uint4 *>(orow + cc) = make_uint4(0, 0, 0, 0);
    }
  }
  tc05_fence_before();
  __syncthreads();
  tc05_fence_after();
  if (warp == 8) tmem_dealloc(tmem, kPtcTmemCols);
}

}  // namespace msa
