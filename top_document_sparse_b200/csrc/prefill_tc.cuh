// prefill_tc.cuh -- multi-token (prefill) sparse GQA attention on the
// 5th-generation tensor cores (MSA, b-lab.team summary item 1 "Scalable Sparse
// Attention" and "Global RoPE", stage "Sparse Generation"): the call's tokens
// attend over [pooled K/V of the retrieved documents' chunks, rank order, all
// visible] ++ [local cache rows, causal: token t sees local rows up to
// cache_len + t], with Q rotated at pos_offset + cache_len + t.
//
// One CTA per (query, kv head, tile of 128 query rows); a row is a (token,
// query head of the GQA group) pair, so a tile holds 128 / G tokens.  The
// context streams through in blocks of 64 rows:
//   S   = Q K^T           tcgen05.mma, M = 128 query rows, N = 64 context
//                          rows, K = D; Q and the K block in shared memory
//                          (K-major, 128-byte swizzle), S in TMEM
//   P   = exp2(S - m)     the four softmax warps: warp w reads TMEM lanes
//                          32w..32w+31 (thread = query row), masks, keeps the
//                          row's reference max m and sum l, writes P as bf16
//                          to shared memory (K-major; over the block's K
//                          rows, dead once S is computed) and, when the row's
//                          max rises more than 8 (log2 units) above m, moves
//                          m and rescales its row of O in TMEM; below that P
//                          stays under 2^8 and the result is the same
//   O  += P V             tcgen05.mma, M = 128, N = D, K = 64 context rows; V
//                          read MN-major straight from its row-major block
// Warp 4 allocates TMEM (64 columns of S, 128 of O) and one lane issues the
// MMAs; every thread loads context blocks (cp.async, two stages) and the
// rotated Q tile.  The softmax warps write O / l at the end.  Every mbarrier
// wait is bounded: on timeout the CTA raises MSA_DEVERR_WAIT_TIMEOUT and skips
// the rest (its outputs are then void), draining issued MMAs before TMEM is
// freed.
#pragma once
#include "attend.cuh"
#include "tc05.cuh"

namespace msa {

constexpr int kPtcRows = 128;             // query rows per tile (UMMA M)
constexpr int kPtcBlk = 64;               // context rows per block (UMMA N of S, K of P V)
constexpr int kPtcThreads = 160;          // warps 0-3 softmax / loads, warp 4 MMA
constexpr uint32_t kPtcTmemCols = 256;    // S at [0, 64), O at [128, 256)

template <int D>
struct PtcSmem {
  static constexpr int kPanels = D / 64;
  static constexpr int kQBytes = kPanels * kPtcRows * 128;   // [panel][128 rows][128 B]
  static constexpr int kKVBytes = kPanels * kPtcBlk * 128;   // [panel][64 rows][128 B]
  static constexpr int kPBytes = kPtcRows * 128;             // [128 rows][64 ctx x 2 B]
  static constexpr int kStage = 2 * kKVBytes;                // K (later P) then V
  static_assert(kPBytes <= kKVBytes, "P takes the place of the block's K rows");
  // Q | 2 stages | bars (s, o, drain) + TMEM slot + flag | chunk table
  static constexpr int kFixed = 1024 + kQBytes + 2 * kStage + 64 + (2 * kMaxTopK + 1) * 4;
  static int bytes(int table_cap) { return kFixed + table_cap * 4; }
};

// Byte offset of 16-byte chunk c (0 .. D/8) of row r of a [panel][rows][128 B]
// tile of `rows` rows (128-byte swizzle: chunk index XOR row % 8).
__device__ __forceinline__ uint32_t ptc_swz(int r, int c, int rows) {
  return static_cast<uint32_t>((c >> 3) * (rows * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// grid (B * H_kv, ceil(T * G / 128)), block kPtcThreads.  append_kernel has
// written the call's rows to the cache before this kernel runs.
template <int D, int G>
__global__ void __launch_bounds__(kPtcThreads, 2)
attend_prefill_tc_kernel(const __nv_bfloat16 *__restrict__ content,
                         const int32_t *__restrict__ ids, int k,
                         const int64_t *__restrict__ doc_chunk_off, int n_docs,
                         const int32_t *__restrict__ slots, int slot_chunks, int H_kv,
                         const __nv_bfloat16 *__restrict__ Q, int T_tok,
                         const __nv_bfloat16 *__restrict__ K_cache,
                         const __nv_bfloat16 *__restrict__ V_cache,
                         const int32_t *__restrict__ cache_len, int cap, int pos_offset,
                         const float2 *__restrict__ rope, float scale_log2, int table_cap,
                         __nv_bfloat16 *__restrict__ O) {
  static_assert(D == 128, "the tensor-core prefill takes head_dim 128");
  static_assert(G >= 1 && G <= 16 && kPtcRows % G == 0, "GQA group");
  using Sm = PtcSmem<D>;
  constexpr int CPR = D / 8;        // 16-byte chunks per row
  constexpr int TT = kPtcRows / G;  // tokens per tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *qs = sm;
  uint8_t *stage0 = qs + Sm::kQBytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(stage0 + 2 * Sm::kStage);  // s, o, drain
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 3);
  volatile int *fail = reinterpret_cast<volatile int *>(tmem_slot + 1);
  int *pre = reinterpret_cast<int *>(bars + 8);
  int *base = pre + (kMaxTopK + 1);
  int *table = base + kMaxTopK;
  const uint32_t bar_s = smem_u32(bars), bar_o = smem_u32(bars + 1), bar_drain = smem_u32(bars + 2);

  const int H_q = H_kv * G;
  const int b = blockIdx.x / H_kv, g = blockIdx.x % H_kv;
  const int t0 = blockIdx.y * TT;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t kv = static_cast<int64_t>(H_kv) * D;
  const int half = D / 2;

  if (threadIdx.x == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    mbar_init(bar_drain, 1);
    *fail = 0;
    fence_mbar_init();
  }
  if (warp == 4) tmem_alloc(smem_u32(tmem_slot), kPtcTmemCols);
  griddep_wait();
  griddep_launch();
  const int len0 = cache_len[b];
  const int n_mem = build_chunk_table(ids + static_cast<int64_t>(b) * k, k, doc_chunk_off, n_docs,
                                      slots ? slots + static_cast<int64_t>(b) * k : nullptr,
                                      slot_chunks, table, pre, base, table_cap);
  // (build_chunk_table ends with __syncthreads: the barriers and the TMEM slot are visible)
  tc05_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_s = tmem, tmem_o = tmem + 128;
  const int t_last = min(t0 + TT, T_tok) - 1;
  const int n_loc = max(0, min(len0 + t_last + 1, cap));
  const int n_ctx = n_mem + n_loc;
  const int nblk = (n_ctx + kPtcBlk - 1) / kPtcBlk;

  auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
    if (*fail) return false;
    if (mbar_wait(bar, parity)) return true;
    *fail = 1;
    raise_device_error(MSA_DEVERR_WAIT_TIMEOUT);
    return false;
  };

  // context block j (rows j*64 ..) into stage s: K and V rows, zero past the context
  auto issue = [&](int j, int s) {
    uint8_t *kb = stage0 + s * Sm::kStage;
    uint8_t *vb = kb + Sm::kKVBytes;
    for (int idx = threadIdx.x; idx < kPtcBlk * CPR; idx += kPtcThreads) {
      const int r = idx / CPR, c = idx % CPR;
      const int x = j * kPtcBlk + r;
      const bool ok = x < n_ctx;
      const __nv_bfloat16 *ksrc = K_cache, *vsrc = V_cache;
      if (ok) {
        if (x < n_mem) {
          ksrc = content + static_cast<int64_t>(table[x]) * 2 * kv + g * D;
          vsrc = ksrc + kv;
        } else {
          const int64_t row = (static_cast<int64_t>(b) * cap + (x - n_mem)) * kv + g * D;
          ksrc = K_cache + row;
          vsrc = V_cache + row;
        }
      }
      cp_async_16(smem_u32(kb + ptc_swz(r, c, kPtcBlk)), ksrc + c * 8, ok);
      cp_async_16(smem_u32(vb + ptc_swz(r, c, kPtcBlk)), vsrc + c * 8, ok);
    }
    cp_async_commit();
  };
  if (nblk > 0) issue(0, 0);
  if (nblk > 1) issue(1, 1);

  // the tile's rotated query rows (row r = token t0 + r / G, head g * G + r % G), in 16-byte
  // pieces: item (token, chunk c of the lower half) rotates elements [8c, 8c + 8) with
  // [half + 8c, half + 8c + 8) of the token's G heads, one RoPE load for all of them, every
  // load of a batch of heads issued before its stores.  Rows past the call's tokens or the
  // cache are zero.
  {
    constexpr int HC = D / 16;         // 16-byte chunks in half a row
    constexpr int GB = G < 4 ? G : 4;  // heads per batch of loads
    for (int it = threadIdx.x; it < TT * HC; it += kPtcThreads) {
      const int tt = it / HC, c = it % HC, t = t0 + tt;
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
          lo[h] = live ? __ldg(reinterpret_cast<const uint4 *>(q0 + (h0 + h) * D)) : make_uint4(0, 0, 0, 0);
          hi[h] = live ? __ldg(reinterpret_cast<const uint4 *>(q0 + (h0 + h) * D + half))
                       : make_uint4(0, 0, 0, 0);
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
          *reinterpret_cast<uint4 *>(qs + ptc_swz(r, c, kPtcRows)) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
          *reinterpret_cast<uint4 *>(qs + ptc_swz(r, c + HC, kPtcRows)) =
              make_uint4(wh[0], wh[1], wh[2], wh[3]);
        }
      }
    }
  }

  // softmax state of this thread's row (warps 0-3)
  const int r = threadIdx.x;  // (valid for warps 0-3: the TMEM lane of the row)
  const int t_row = t0 + r / G;
  const int vis = n_mem + len0 + t_row;  // last visible context index of the row
  float m_run = -INFINITY, l_run = 0.0f;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  constexpr uint32_t idesc_s = umma_idesc_bf16_f32<kPtcRows, kPtcBlk>();
  constexpr uint32_t idesc_o = umma_idesc_bf16_f32_bmn<kPtcRows, D>();

  for (int j = 0; j < nblk; ++j) {
    const int st = j & 1;
    uint8_t *kb = stage0 + st * Sm::kStage;
    uint8_t *vb = kb + Sm::kKVBytes;
    uint8_t *psm = kb;  // P [128 rows][64 context] bf16, once S = Q K^T is computed
    if (j + 1 < nblk) cp_async_wait<1>(); else cp_async_wait<0>();
    fence_proxy_async_smem();  // the copies (and Q) become visible to the tensor cores
    tc05_fence_before();
    __syncthreads();  // (A) block j is in shared memory
    tc05_fence_after();
    if (warp == 4 && lane == 0 && !*fail) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t pa = static_cast<uint32_t>((kk >> 2) * kPtcRows * 128 + (kk & 3) * 32);
        const uint32_t pb = static_cast<uint32_t>((kk >> 2) * kPtcBlk * 128 + (kk & 3) * 32);
        umma_bf16(tmem_s, umma_desc_k_sw128(smem_u32(qs) + pa), umma_desc_k_sw128(smem_u32(kb) + pb),
                  idesc_s, kk != 0);
      }
      umma_commit(bar_s);
    }
    if (warp < 4) {
      const bool ok = wait(bar_s, j & 1);
      const bool okw = __all_sync(0xffffffffu, ok);
      tc05_fence_after();
      // the row's last visible context index, relative to this block (-1: nothing)
      const int lim = okw ? min(vis, n_ctx - 1) - j * kPtcBlk : -1;
      float s[kPtcBlk];
      static_assert(kPtcBlk == 64, "one 64-column TMEM load per block");
      if (okw) tmem_ld64(tmem_s + lane_base, s);
      if (lim < kPtcBlk - 1) {  // a diagonal block (or the context's ragged end): mask
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
      for (int c = 0; c < kPtcBlk; c += 8) {
        float pv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          pv[i] = ex2_approx(fmaf(s[c + i], scale_log2, -mo));
          ps[i & 3] += pv[i];
        }
        uint4 w;
        w.x = pack_bf16x2(pv[0], pv[1]);
        w.y = pack_bf16x2(pv[2], pv[3]);
        w.z = pack_bf16x2(pv[4], pv[5]);
        w.w = pack_bf16x2(pv[6], pv[7]);
        // (the previous block's P V completed before this block began: P is free)
        *reinterpret_cast<uint4 *>(psm + ptc_swz(r, c / 8, kPtcRows)) = w;
      }
      const float psum = (ps[0] + ps[1]) + (ps[2] + ps[3]);
      l_run = l_run * alpha + psum;
      m_run = m_new;
      // O's row: rescale when the max rose (the previous block's P V has completed).  The
      // TMEM loads and stores are warp-collective: the warp takes them when any of its rows
      // needs it, each thread with its own factor (1 where nothing rose).
      if (j > 0 && okw && __any_sync(0xffffffffu, alpha < 1.0f)) {
#pragma unroll 1
        for (int c = 0; c < D; c += 16) {
          float x[16];
          tmem_ld16(tmem_o + lane_base + c, x);
#pragma unroll
          for (int i = 0; i < 16; ++i) x[i] *= alpha;
          tmem_st16(tmem_o + lane_base + c, x);
        }
      }
      fence_proxy_async_smem();  // P becomes visible to the tensor cores
      tc05_fence_before();
    }
    __syncthreads();  // (B) P and O are ready for this block's P V
    tc05_fence_after();
    if (warp == 4 && lane == 0 && !*fail) {
#pragma unroll
      for (int ks = 0; ks < kPtcBlk / 16; ++ks)
        umma_bf16(tmem_o, umma_desc_k_sw128(smem_u32(psm) + ks * 32),
                  umma_desc_mn_sw128(smem_u32(vb) + ks * 16 * 128, Sm::kKVBytes / Sm::kPanels),
                  idesc_o, (j | ks) != 0);
      umma_commit(bar_o);
    }
    // every thread: the P V of this block must finish before P and this stage are reused
    wait(bar_o, j & 1);
    tc05_fence_after();
    if (j + 2 < nblk) issue(j + 2, st);
  }

  // O / l for the rows of this call's tokens (the TMEM loads by whole warps)
  const bool row_out = warp < 4 && t_row <= t_last && t_row < T_tok;
  const bool have_o = warp < 4 && nblk > 0 && __all_sync(0xffffffffu, !*fail);
  if (have_o) {
    const bool live = len0 + t_row < cap && l_run > 0.0f;
    const float inv = live ? 1.0f / l_run : 0.0f;
    __nv_bfloat16 *orow = O + ((static_cast<int64_t>(b) * T_tok + t_row) * H_q + g * G + r % G) * D;
#pragma unroll 1
    for (int c = 0; c < D; c += 16) {
      float x[16];
      tmem_ld16(tmem_o + lane_base + c, x);
      if (!row_out) continue;
      uint4 w0, w1;
      w0.x = pack_bf16x2(x[0] * inv, x[1] * inv);
      w0.y = pack_bf16x2(x[2] * inv, x[3] * inv);
      w0.z = pack_bf16x2(x[4] * inv, x[5] * inv);
      w0.w = pack_bf16x2(x[6] * inv, x[7] * inv);
      w1.x = pack_bf16x2(x[8] * inv, x[9] * inv);
      w1.y = pack_bf16x2(x[10] * inv, x[11] * inv);
      w1.z = pack_bf16x2(x[12] * inv, x[13] * inv);
      w1.w = pack_bf16x2(x[14] * inv, x[15] * inv);
      *reinterpret_cast<uint4 *>(orow + c) = w0;
      *reinterpret_cast<uint4 *>(orow + c + 8) = w1;
    }
  } else if (row_out) {
    __nv_bfloat16 *orow = O + ((static_cast<int64_t>(b) * T_tok + t_row) * H_q + g * G + r % G) * D;
    for (int c = 0; c < D; c += 8) *reinterpret_cast<uint4 *>(orow + c) = make_uint4(0, 0, 0, 0);
  }
  tc05_fence_before();
  __syncthreads();
  tc05_fence_after();
  if (warp == 4) {
    if (lane == 0) {  // every MMA issued here has completed before TMEM is freed
      umma_commit(bar_drain);
      mbar_wait(bar_drain, 0);
    }
    __syncwarp();
    tmem_dealloc(tmem, kPtcTmemCols);
  }
}

}  // namespace msa
