// msa.cu -- the C ABI of libmsa.so (declared in include/msa.h): host-side
// validation and orchestration of the MSA kernels.  Every kernel lives in the
// headers included below; this file is the single translation unit.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <utility>

#include "attend.cuh"
#include "backward.cuh"
#include "prefill_tc.cuh"
#include "common.cuh"
#include "pool.cuh"
#include "route.cuh"
#include "route_tc.cuh"
#include "tier.cuh"
#include "topk.cuh"

// Scratch of msa_sparse_attend_static: a fixed device array, so that callers
// which cannot allocate device memory still get the split-context attention.
// Every GPU that loads the library holds these 4 MiB until the process exits.
static constexpr size_t kStaticAttendScratchBytes = size_t(4) << 20;
static __device__ __align__(256) uint8_t g_attend_static_scratch[kStaticAttendScratchBytes];

namespace {

thread_local std::string g_last_error;

msa_status fail(msa_status s, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

msa_status cuda_fail(cudaError_t e, const char *what) {
  return fail(MSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define MSA_CUDA(call)                                 \
  do {                                                 \
    cudaError_t e_ = (call);                           \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
  } while (0)

// Every kernel launch is followed by MSA_LAUNCHED: it checks the launch and
// counts it (msa_launch_count).
std::atomic<uint64_t> g_launches{0};

#define MSA_LAUNCHED(what)                              \
  do {                                                  \
    cudaError_t e_ = cudaGetLastError();                \
    if (e_ != cudaSuccess) return cuda_fail(e_, what);  \
    g_launches.fetch_add(1, std::memory_order_relaxed); \
  } while (0)

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel on the stream drains (it calls griddep_wait() before
// its first global memory access), which hides the launch and the kernel's
// setup behind the previous kernel's tail.  Used for the per-token decode
// path, where a step is a chain of short dependent kernels.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Same, with thread-block clusters of cluster_x CTAs along x (1: none).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                               cudaStream_t st, unsigned cluster_x, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cluster_x > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Device address of the static attention scratch on the current device, looked
// up once per device (cudaGetSymbolAddress with that device current).
msa_status static_attend_scratch(void **out) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void *addr[kMaxDevices] = {};
  int dev = 0;
  MSA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(MSA_ERR_UNSUPPORTED, "device %d", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_attend_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static attention scratch)");
    addr[dev] = p;
  }
  *out = addr[dev];
  return MSA_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
int round32(int x) { return (x + 31) / 32 * 32; }

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

int max_dyn_smem() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (n <= 0) n = 232448;
  }
  return n;
}

// ---------------------------------------------------------------- TMA maps
PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 map over a row-major [rows][cols] array, box {64 cols, box_rows},
// 128-byte swizzle, out-of-range rows read as zero.
msa_status make_map_bf16(CUtensorMap *map, const void *base, int64_t rows, int64_t cols,
                         int box_rows) {
  auto fn = encode_tiled();
  if (!fn) return fail(MSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MSA_OK;
}

// 3-D bf16 map over [d2][d1][d0] with the given byte strides of dimensions 1 and 2, box
// {64, box1, box2}, 128-byte swizzle, out-of-range elements read as zero.
msa_status make_map_bf16_3d(CUtensorMap *map, const void *base, int64_t d0, int64_t d1, int64_t d2,
                            int64_t stride1, int64_t stride2, int box1, int box2) {
  auto fn = encode_tiled();
  if (!fn) return fail(MSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d0), static_cast<cuuint64_t>(d1),
                        static_cast<cuuint64_t>(d2)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(stride1), static_cast<cuuint64_t>(stride2)};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box1), static_cast<cuuint32_t>(box2)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MSA_OK;
}

// ---------------------------------------------------------------- helpers
size_t elem_size(msa_dtype t) { return t == MSA_BF16 ? 2 : 4; }

int topk_splits(int n_docs) { return (n_docs + msa::kTopkSlice - 1) / msa::kTopkSlice; }

// Context splits of one attention launch: enough CTAs for about three per
// SM (the kernel holds four); more splits only add per-CTA fixed cost and
// combine traffic (measured on the 1M- and 100M-token decode workloads).
int attend_splits(int B, int T, int H_kv, int64_t max_ctx) {
  const int64_t ctas = static_cast<int64_t>(B) * T * H_kv;
  const int64_t want = 3LL * num_sms();
  if (ctas >= want) return 1;
  int64_t s = (want + ctas - 1) / ctas;
  const int64_t by_len = std::max<int64_t>(1, (max_ctx + 63) / 64);
  return static_cast<int>(std::min<int64_t>(std::min<int64_t>(s, by_len), 32));
}

struct AttendPlan {
  int n_split = 1;
  int table_cap = 0;
  int early = 0;  // the local part may start before the wait for the previous kernel
  size_t part_o = 0, part_ml = 0;  // byte offsets in the workspace
  size_t bytes = 0;
};

AttendPlan plan_attend(const msa_memory *mem, int B, int T, int k, int H_q, int cap) {
  AttendPlan p;
  const int64_t max_mem = static_cast<int64_t>(k) * mem->max_doc_chunks;
  p.table_cap = static_cast<int>(std::min<int64_t>(max_mem, msa::kMaxMemRows));
  if (mem->dtype != MSA_BF16) return p;
  p.n_split = attend_splits(B, T, mem->H_kv, max_mem + cap);
  if (p.n_split > 1) {
    const size_t rows = static_cast<size_t>(B) * T * H_q * p.n_split;
    p.part_o = 0;
    p.part_ml = round256(rows * mem->D * 4);
    p.bytes = p.part_ml + round256(rows * 2 * 4);
  }
  return p;
}

struct RoutePlan {
  size_t qhat = 0, cand = 0, bytes = 0;
  int n_split = 1;
};

RoutePlan plan_route(const msa_memory *mem, int B, int T, int k) {
  RoutePlan p;
  const size_t W = static_cast<size_t>(mem->H_r) * mem->d_r;
  p.qhat = 0;
  p.cand = round256(static_cast<size_t>(B) * T * W * elem_size(mem->dtype));
  p.n_split = topk_splits(mem->n_docs);
  p.bytes = p.cand + (p.n_split > 1 ? round256(static_cast<size_t>(B) * p.n_split * k * 8) : 0);
  return p;
}

// NT = 64 query rows stream their feature slices with the key slices (a
// resident 64-row tile would leave only four ring stages); narrower tiles
// stay resident.
template <int NT, bool QS = (NT >= 64)>
msa_status launch_route_tc(const msa_memory *mem, const void *keys, const void *qhat, int R, int T,
                           float *state, cudaStream_t st, int ctas_per_sm = 1) {
  using L = msa::RouteTcLayout<NT, QS>;
  const int W = mem->H_r * mem->d_r;
  CUtensorMap tmK, tmQ;
  msa_status s = make_map_bf16(&tmK, keys, mem->n_chunks, W, L::kTileC);
  if (s != MSA_OK) return s;
  s = make_map_bf16(&tmQ, qhat, R, W, NT);
  if (s != MSA_OK) return s;
  // (256 B per CTA left for the epilogue's static shared memory; ~1 KB per CTA reserved)
  const int maxs = ctas_per_sm == 1 ? max_dyn_smem() : 233472 / ctas_per_sm - 1024 - 256;
  int stages = 12;
  while (stages > 2 && L::bytes(W, stages) + 256 > static_cast<size_t>(maxs)) --stages;
  const size_t smem = L::bytes(W, stages);
  if (smem + 256 > static_cast<size_t>(maxs))
    return fail(MSA_ERR_UNSUPPORTED, "router width %d needs %zu B of shared memory", W, smem);
  auto kern = msa::route_tc_kernel<NT, QS>;
  MSA_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  const int n_ct = static_cast<int>((mem->n_chunks + L::kTileC - 1) / L::kTileC);
  const int n_rt = (R + NT - 1) / NT;
  const int64_t n_tiles = static_cast<int64_t>(n_ct) * n_rt;
  if (n_tiles > INT32_MAX) return fail(MSA_ERR_UNSUPPORTED, "too many route tiles");
  const int grid = static_cast<int>(std::min<int64_t>(n_tiles, static_cast<int64_t>(num_sms()) * ctas_per_sm));
  MSA_CUDA(launch_pdl(kern, dim3(grid), dim3(192), smem, st, tmK, tmQ, mem->n_chunks, R, W, T,
                      1.0f / mem->H_r, mem->d_chunk_doc, mem->n_docs, state, n_ct,
                      static_cast<int>(n_tiles), stages));
  MSA_LAUNCHED("route_tc_kernel");
  return MSA_OK;
}

template <int KL>
msa_status launch_topk(const msa_memory *mem, const float *state, const uint8_t *exclude, int B,
                       int k, int n_split, unsigned long long *cand, int32_t *ids, float *scores,
                       cudaStream_t st) {
  if (n_split == 1 && mem->n_docs <= 128 * msa::kTopkPerThread) {
    MSA_CUDA(launch_pdl(msa::topk_partial_kernel<KL, 128>, dim3(1, B), dim3(128), 0, st, state,
                        exclude, mem->n_docs, k, 1, cand, ids, scores));
  } else {
    MSA_CUDA(launch_pdl(msa::topk_partial_kernel<KL>, dim3(n_split, B), dim3(msa::kTopkThreads),
                        0, st, state, exclude, mem->n_docs, k, n_split, cand, ids, scores));
  }
  MSA_LAUNCHED("topk_partial_kernel");
  if (n_split > 1) {
    MSA_CUDA(launch_pdl(msa::topk_merge_kernel<KL>, dim3(B), dim3(msa::kTopkThreads), 0, st,
                        static_cast<const unsigned long long *>(cand), n_split * k, k, ids, scores));
    MSA_LAUNCHED("topk_merge_kernel");
  }
  return MSA_OK;
}

// q_early: Qr is the caller's (written by no kernel of this library), so the query
// normalisation may read it before the previous kernel completes.
msa_status route_impl(const msa_memory *mem, const void *keys, const void *Qr, int B, int T, int k,
                      const uint8_t *exclude, float *state, int32_t *ids, float *scores,
                      void *ws, size_t ws_bytes, cudaStream_t st, int q_pitch = 0,
                      bool q_early = false) {
  if (q_pitch <= 0) q_pitch = T;
  if (!mem) return fail(MSA_ERR_INVALID_ARG, "null memory");
  if (B < 1 || T < 0) return fail(MSA_ERR_INVALID_ARG, "batch must be >= 1 and tokens >= 0");
  if (k < 1 || k > mem->n_docs || k > msa::kMaxTopK)
    return fail(MSA_ERR_INVALID_ARG, "k=%d must be in [1, min(n_docs=%d, %d)]", k, mem->n_docs,
                msa::kMaxTopK);
  if (!state || !ids || !scores) return fail(MSA_ERR_INVALID_ARG, "null state/ids/scores");
  if (T > 0 && (!keys || !Qr)) return fail(MSA_ERR_INVALID_ARG, "null router keys or Qr");
  if (!aligned16(keys) || !aligned16(Qr) || !aligned16(ws))
    return fail(MSA_ERR_INVALID_ARG, "router keys, Qr and workspace must be 16-byte aligned");
  const RoutePlan plan = plan_route(mem, B, T, k);
  if (plan.n_split * k > msa::kTopkSlice)
    return fail(MSA_ERR_UNSUPPORTED, "top-k merge of %d candidates is too large",
                plan.n_split * k);
  if (ws_bytes < plan.bytes || (plan.bytes > 0 && !ws))
    return fail(MSA_ERR_INVALID_ARG, "workspace too small: %zu < %zu", ws_bytes, plan.bytes);
  const int64_t R64 = static_cast<int64_t>(B) * T;
  if (R64 > INT32_MAX / 2) return fail(MSA_ERR_UNSUPPORTED, "too many query rows");
  const int R = static_cast<int>(R64);
  const int W = mem->H_r * mem->d_r;
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  if (R > 0) {
    const int thr = round32(W / 4);
    if (mem->dtype == MSA_BF16) {
      auto *qh = reinterpret_cast<__nv_bfloat16 *>(wsb + plan.qhat);
      MSA_CUDA(launch_pdl(msa::qnorm_kernel<__nv_bfloat16>, dim3(R), dim3(thr), 0, st,
                          static_cast<const __nv_bfloat16 *>(Qr), W, mem->d_r, T, q_pitch, qh,
                          q_early ? 1 : 0));
      MSA_LAUNCHED("qnorm_kernel");
      msa_status s;
      if (R <= 16)
        s = launch_route_tc<16>(mem, keys, qh, R, T, state, st);
      else if (R <= 32)
        s = launch_route_tc<32>(mem, keys, qh, R, T, state, st);
      else if (R <= 64)
        s = launch_route_tc<32, true>(mem, keys, qh, R, T, state, st, 2);
      else if (R <= 128)
        s = launch_route_tc<64>(mem, keys, qh, R, T, state, st);
      else  // many rows (prefill, interleave rounds): 128-row tiles re-read each key slice half as often
        s = launch_route_tc<128, true>(mem, keys, qh, R, T, state, st);
      if (s != MSA_OK) return s;
    } else {
      auto *qh = reinterpret_cast<float *>(wsb + plan.qhat);
      msa::qnorm_kernel<float><<<R, thr, 0, st>>>(static_cast<const float *>(Qr), W, mem->d_r, T,
                                                  q_pitch, qh, 0);
      MSA_LAUNCHED("qnorm_kernel");
      dim3 grid(static_cast<unsigned>((mem->n_chunks + 31) / 32), static_cast<unsigned>((R + 31) / 32));
      if (grid.y > 65535) return fail(MSA_ERR_UNSUPPORTED, "too many query rows for fp32 route");
      msa::route_simt_kernel<float><<<grid, 256, 0, st>>>(
          static_cast<const float *>(keys), qh, mem->n_chunks, R, W, T, 1.0f / mem->H_r,
          mem->d_chunk_doc, mem->n_docs, state);
      MSA_LAUNCHED("route_simt_kernel");
    }
  }
  auto *cand = reinterpret_cast<unsigned long long *>(wsb + plan.cand);
  if (B > 65535) return fail(MSA_ERR_UNSUPPORTED, "batch too large for top-k");
  if (k <= 16) return launch_topk<16>(mem, state, exclude, B, k, plan.n_split, cand, ids, scores, st);
  if (k <= 32) return launch_topk<32>(mem, state, exclude, B, k, plan.n_split, cand, ids, scores, st);
  return launch_topk<64>(mem, state, exclude, B, k, plan.n_split, cand, ids, scores, st);
}

// The tensor-core prefill (head_dim 128, bf16) with a K/V ring of NS stages.
template <int G, int NS>
msa_status launch_prefill_tc(const msa_memory *mem, const void *content, const int32_t *ids,
                             const int32_t *slots, int slot_chunks, int B, int k, int T,
                             const void *Q, void *Kc, void *Vc, int32_t *cache_len, int cap,
                             int pos_offset, float scale_log2, const AttendPlan &plan, void *O,
                             cudaStream_t st) {
  constexpr int D = 128;
  const int smem_pt = msa::PtcSmem<D, NS>::bytes(plan.table_cap);
  // the local cache as [B * cap rows][H_kv][D]: box {64 of D, head g, 64 rows}
  CUtensorMap tm_k, tm_v;
  const int64_t row_bytes = static_cast<int64_t>(mem->H_kv) * D * 2;
  msa_status ms = make_map_bf16_3d(&tm_k, Kc, D, mem->H_kv, static_cast<int64_t>(B) * cap,
                                   D * 2, row_bytes, 1, msa::kPtcBlk);
  if (ms != MSA_OK) return ms;
  ms = make_map_bf16_3d(&tm_v, Vc, D, mem->H_kv, static_cast<int64_t>(B) * cap, D * 2,
                        row_bytes, 1, msa::kPtcBlk);
  if (ms != MSA_OK) return ms;
  auto kpt = msa::attend_prefill_tc_kernel<128, G, NS>;
  MSA_CUDA(cudaFuncSetAttribute(kpt, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_pt));
  constexpr int TT = msa::kPtcRows / G;
  const int n_tiles = (T + TT - 1) / TT;
  const int n_pairs = (n_tiles + 1) / 2;
  const int64_t n_ctas = static_cast<int64_t>(n_pairs) * B * mem->H_kv;
  if (n_ctas > 0x7FFFFFFF) return fail(MSA_ERR_UNSUPPORTED, "too many query tokens");
  dim3 grid_pt(static_cast<unsigned>(n_ctas));
  MSA_CUDA(launch_pdl(kpt, grid_pt, dim3(msa::kPtcThreads), smem_pt, st,
                      static_cast<const __nv_bfloat16 *>(content), ids, k,
                      static_cast<const int64_t *>(mem->d_doc_chunk_off), mem->n_docs, slots,
                      slot_chunks, mem->H_kv, static_cast<const __nv_bfloat16 *>(Q), T,
                      static_cast<const __nv_bfloat16 *>(Kc),
                      static_cast<const __nv_bfloat16 *>(Vc),
                      static_cast<const int32_t *>(cache_len), cap, pos_offset,
                      static_cast<const float2 *>(mem->d_rope), scale_log2, plan.table_cap,
                      static_cast<__nv_bfloat16 *>(O), tm_k, tm_v, n_pairs));
  MSA_LAUNCHED("attend_prefill_tc_kernel");
  MSA_CUDA(launch_pdl(msa::advance_kernel, dim3((B + 255) / 256), dim3(256), 0, st, cache_len,
                      B, T, cap));
  MSA_LAUNCHED("advance_kernel");
  return MSA_OK;
}

template <int D, int G>
msa_status launch_attend_mma(const msa_memory *mem, const void *content, const int32_t *ids,
                             const int32_t *slots, int slot_chunks, int B, int k, int T,
                             const void *Q, const void *K_new, const void *V_new, void *Kc,
                             void *Vc, int32_t *cache_len, int cap, int pos_offset,
                             const AttendPlan &plan, void *O, void *ws, cudaStream_t st) {
  const float scale_log2 = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)) * 1.4426950408889634);
  if constexpr (D == 128) {
    // several tokens (prefill), tensor cores: one CTA per (query, kv head, pair of adjacent
    // tiles of 128 / G tokens x G heads), a K/V ring of three stages (four measured slower:
    // 265 against 247 us at the 1M prefill); append_kernel ran before
    if (T > 1) {
      if (msa::PtcSmem<D, 3>::bytes(plan.table_cap) <= max_dyn_smem())
        return launch_prefill_tc<G, 3>(mem, content, ids, slots, slot_chunks, B, k, T, Q, Kc, Vc,
                                       cache_len, cap, pos_offset, scale_log2, plan, O, st);
    }
  }
  if (T > 1) {
    // several tokens (prefill) on mma.sync (head_dim 64, or a chunk table too large for the
    // tensor-core kernel's shared memory): one CTA per (query, kv head, tile of 4 x 16 / G
    // tokens) shares each staged context block between its tokens; append_kernel ran before
    using Pf = msa::PfSmem<D>;
    const int smem_pf = Pf::bytes(plan.table_cap);
    auto kpf = msa::attend_prefill_kernel<D, G>;
    MSA_CUDA(cudaFuncSetAttribute(kpf, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_pf));
    constexpr int TC = msa::kPfWarps * (16 / G);
    dim3 grid_pf(static_cast<unsigned>(B * mem->H_kv), static_cast<unsigned>((T + TC - 1) / TC));
    if (grid_pf.y > 65535) return fail(MSA_ERR_UNSUPPORTED, "too many query tokens");
    MSA_CUDA(launch_pdl(kpf, grid_pf, dim3(32 * msa::kPfWarps), smem_pf, st,
                        static_cast<const __nv_bfloat16 *>(content), ids, k,
                        static_cast<const int64_t *>(mem->d_doc_chunk_off), mem->n_docs, slots,
                        slot_chunks, mem->H_kv, static_cast<const __nv_bfloat16 *>(Q), T,
                        static_cast<const __nv_bfloat16 *>(Kc), static_cast<const __nv_bfloat16 *>(Vc),
                        static_cast<const int32_t *>(cache_len), cap, pos_offset,
                        static_cast<const float2 *>(mem->d_rope), scale_log2, plan.table_cap,
                        static_cast<__nv_bfloat16 *>(O)));
    MSA_LAUNCHED("attend_prefill_kernel");
    MSA_CUDA(launch_pdl(msa::advance_kernel, dim3((B + 255) / 256), dim3(256), 0, st, cache_len, B,
                        T, cap));
    MSA_LAUNCHED("advance_kernel");
    return MSA_OK;
  }
  using Sm = msa::AttSmem<D>;
  const int smem = Sm::bytes(plan.table_cap);
  auto kern = msa::attend_mma_kernel<D, G>;
  MSA_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  uint8_t *wsb = static_cast<uint8_t *>(ws);
  float *part_o = plan.n_split > 1 ? reinterpret_cast<float *>(wsb + plan.part_o) : nullptr;
  float *part_ml = plan.n_split > 1 ? reinterpret_cast<float *>(wsb + plan.part_ml) : nullptr;
  const int fuse_append = 1;  // (T == 1 here)
  // One token, one split: the H_kv CTAs of a query form a cluster, and the
  // kernel advances cache_len itself once all of them have read it (cluster
  // barrier), so no advance kernel follows.
  const int cluster_advance = (T == 1 && plan.n_split == 1 && mem->H_kv <= 8) ? 1 : 0;
  dim3 grid(static_cast<unsigned>(B * mem->H_kv), plan.n_split, T);
  MSA_CUDA(launch_pdl_cluster(
      kern, grid, dim3(32 * msa::kAttWarps), smem, st,
      static_cast<unsigned>(cluster_advance ? mem->H_kv : 1),
      static_cast<const __nv_bfloat16 *>(content), ids, k,
      static_cast<const int64_t *>(mem->d_doc_chunk_off), mem->n_docs, slots, slot_chunks,
      mem->H_kv, static_cast<const __nv_bfloat16 *>(Q), T, static_cast<__nv_bfloat16 *>(Kc),
      static_cast<__nv_bfloat16 *>(Vc), static_cast<const __nv_bfloat16 *>(K_new),
      static_cast<const __nv_bfloat16 *>(V_new), cache_len, cap, pos_offset,
      static_cast<const float2 *>(mem->d_rope), scale_log2, plan.n_split, plan.table_cap,
      fuse_append, plan.early, cluster_advance, static_cast<__nv_bfloat16 *>(O), part_o,
      part_ml));
  MSA_LAUNCHED("attend_mma_kernel");
  if (plan.n_split > 1) {
    // merge the splits and advance cache_len (every attention CTA has read it)
    MSA_CUDA(launch_pdl(msa::attend_combine_kernel,
                        dim3(static_cast<unsigned>(static_cast<int64_t>(B) * T * mem->H_kv * G)),
                        dim3(D), 0, st, static_cast<const float *>(part_o),
                        static_cast<const float *>(part_ml), plan.n_split, D,
                        static_cast<__nv_bfloat16 *>(O), cache_len, T * mem->H_kv * G, T, cap));
    MSA_LAUNCHED("attend_combine_kernel");
  } else if (!cluster_advance) {
    MSA_CUDA(launch_pdl(msa::advance_kernel, dim3((B + 255) / 256), dim3(256), 0, st, cache_len, B,
                        T, cap));
    MSA_LAUNCHED("advance_kernel");
  }
  return MSA_OK;
}

template <int D>
msa_status dispatch_group(int G, const msa_memory *mem, const void *content, const int32_t *ids,
                          const int32_t *slots, int slot_chunks, int B, int k, int T,
                          const void *Q, const void *K_new, const void *V_new, void *Kc, void *Vc,
                          int32_t *cache_len, int cap, int pos_offset, const AttendPlan &plan,
                          void *O, void *ws, cudaStream_t st) {
#define MSA_G(g)                                                                                  \
  case g:                                                                                         \
    return launch_attend_mma<D, g>(mem, content, ids, slots, slot_chunks, B, k, T, Q, K_new,      \
                                   V_new, Kc, Vc, cache_len, cap, pos_offset, plan, O, ws, st);
  switch (G) {
    MSA_G(1) MSA_G(2) MSA_G(4) MSA_G(8) MSA_G(16)
    default:
      return fail(MSA_ERR_UNSUPPORTED, "GQA group %d (must be 1, 2, 4, 8 or 16)", G);
  }
#undef MSA_G
}

// Shape checks shared by every attention entry point; they run before any
// scratch is sized or anything is enqueued.
msa_status attend_shape_check(const msa_memory *mem, int B, int k, int T, int H_q, int cap,
                              int pos_offset) {
  if (!mem) return fail(MSA_ERR_INVALID_ARG, "null memory");
  if (B < 1 || T < 1) return fail(MSA_ERR_INVALID_ARG, "batch and tokens must be >= 1");
  if (k < 0 || k > msa::kMaxTopK) return fail(MSA_ERR_INVALID_ARG, "k=%d out of range", k);
  if (H_q < mem->H_kv || H_q % mem->H_kv != 0)
    return fail(MSA_ERR_INVALID_ARG, "n_q_heads=%d must be a multiple of n_kv_heads=%d", H_q,
                mem->H_kv);
  if (H_q > 16 * 32) return fail(MSA_ERR_UNSUPPORTED, "too many query heads");
  if (cap < 1 || pos_offset < 0 ||
      static_cast<int64_t>(pos_offset) + cap > mem->max_local_position)
    return fail(MSA_ERR_INVALID_ARG,
                "pos_offset=%d + cache_capacity=%d must be <= max_local_position=%d", pos_offset,
                cap, mem->max_local_position);
  if (static_cast<int64_t>(k) * mem->max_doc_chunks > msa::kMaxMemRows)
    return fail(MSA_ERR_UNSUPPORTED, "k * max_doc_chunks = %lld exceeds %d retrieved rows",
                (long long)k * mem->max_doc_chunks, msa::kMaxMemRows);
  if (static_cast<int64_t>(B) * T > 2147483647LL / 64)
    return fail(MSA_ERR_UNSUPPORTED, "batch * tokens too large");
  return MSA_OK;
}

msa_status attend_impl(const msa_memory *mem, const void *content, const int32_t *ids,
                       const int32_t *slots, int slot_chunks, int B, int k, int T, int H_q,
                       const void *Q, const void *K_new, const void *V_new, void *K_cache,
                       void *V_cache, int32_t *cache_len, int cap, int pos_offset, void *O,
                       void *ws, size_t ws_bytes, cudaStream_t st, bool early = false) {
  const msa_status chk = attend_shape_check(mem, B, k, T, H_q, cap, pos_offset);
  if (chk != MSA_OK) return chk;
  if (!content || (k > 0 && !ids) || !Q || !K_new || !V_new || !K_cache || !V_cache ||
      !cache_len || !O)
    return fail(MSA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(content) || !aligned16(Q) || !aligned16(K_new) || !aligned16(V_new) ||
      !aligned16(K_cache) || !aligned16(V_cache) || !aligned16(O) || !aligned16(ws))
    return fail(MSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  AttendPlan plan = plan_attend(mem, B, T, k, H_q, cap);
  plan.early = early ? 1 : 0;
  if (ws_bytes < plan.bytes || (plan.bytes > 0 && !ws))
    return fail(MSA_ERR_INVALID_ARG, "workspace too small: %zu < %zu", ws_bytes, plan.bytes);
  const int D = mem->D, H_kv = mem->H_kv;
  if (mem->dtype == MSA_BF16) {
    // one token: the attention kernel appends the new row itself; more: append first
    if (T > 1) {
      const int athr = round32(H_kv * D / 8);
      if (athr > 1024) return fail(MSA_ERR_UNSUPPORTED, "n_kv_heads * head_dim too large");
      msa::append_kernel<__nv_bfloat16><<<B * T, athr, 0, st>>>(
          static_cast<const __nv_bfloat16 *>(K_new), static_cast<const __nv_bfloat16 *>(V_new), T,
          H_kv, D, static_cast<__nv_bfloat16 *>(K_cache), static_cast<__nv_bfloat16 *>(V_cache),
          cache_len, cap, pos_offset, mem->d_rope);
      MSA_LAUNCHED("append_kernel");
    }
    const int G = H_q / H_kv;
    if (D == 128)
      return dispatch_group<128>(G, mem, content, ids, slots, slot_chunks, B, k, T, Q, K_new,
                                 V_new, K_cache, V_cache, cache_len, cap, pos_offset, plan, O, ws,
                                 st);
    return dispatch_group<64>(G, mem, content, ids, slots, slot_chunks, B, k, T, Q, K_new, V_new,
                              K_cache, V_cache, cache_len, cap, pos_offset, plan, O, ws, st);
  }
  // fp32: append, attention, advance
  if (H_q > 16) return fail(MSA_ERR_UNSUPPORTED, "fp32 attention supports <= 16 query heads");
  const int athr = round32(H_kv * D / 8);
  if (athr > 1024) return fail(MSA_ERR_UNSUPPORTED, "n_kv_heads * head_dim too large");
  msa::append_kernel<float><<<B * T, athr, 0, st>>>(
      static_cast<const float *>(K_new), static_cast<const float *>(V_new), T, H_kv, D,
      static_cast<float *>(K_cache), static_cast<float *>(V_cache), cache_len, cap, pos_offset,
      mem->d_rope);
  MSA_LAUNCHED("append_kernel");
  const float scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  const int thr = H_q * 32;
  if (D == 128)
    msa::attend_simt_kernel<float, 128><<<B * T, thr, 0, st>>>(
        static_cast<const float *>(content), ids, k, mem->d_doc_chunk_off, mem->n_docs, slots,
        slot_chunks, H_kv, H_q, static_cast<const float *>(Q), T,
        static_cast<const float *>(K_cache), static_cast<const float *>(V_cache), cache_len, cap,
        pos_offset, mem->d_rope, scale, static_cast<float *>(O));
  else
    msa::attend_simt_kernel<float, 64><<<B * T, thr, 0, st>>>(
        static_cast<const float *>(content), ids, k, mem->d_doc_chunk_off, mem->n_docs, slots,
        slot_chunks, H_kv, H_q, static_cast<const float *>(Q), T,
        static_cast<const float *>(K_cache), static_cast<const float *>(V_cache), cache_len, cap,
        pos_offset, mem->d_rope, scale, static_cast<float *>(O));
  MSA_LAUNCHED("attend_simt_kernel");
  msa::advance_kernel<<<(B + 255) / 256, 256, 0, st>>>(cache_len, B, T, cap);
  MSA_LAUNCHED("advance_kernel");
  return MSA_OK;
}

}  // namespace

// ===================================================================== C ABI
extern "C" {

int32_t msa_version(void) { return 1 * 10000 + 0 * 100 + 0; }

uint64_t msa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char *msa_status_string(msa_status s) {
  switch (s) {
    case MSA_OK: return "ok";
    case MSA_ERR_INVALID_ARG: return "invalid argument";
    case MSA_ERR_UNSUPPORTED: return "unsupported shape";
    case MSA_ERR_CUDA: return "CUDA error";
    case MSA_ERR_OUT_OF_MEMORY: return "out of memory";
    case MSA_ERR_TIMEOUT: return "device wait timed out";
    case MSA_ERR_STATE: return "device bounds check fired";
  }
  return "unknown status";
}

const char *msa_last_error(void) { return g_last_error.c_str(); }

msa_status msa_memory_create(const msa_memory_config *cfg, msa_memory **out) {
  if (!cfg || !out) return fail(MSA_ERR_INVALID_ARG, "null config or output");
  *out = nullptr;
  if (cfg->n_docs < 1 || !cfg->doc_token_offsets)
    return fail(MSA_ERR_INVALID_ARG, "n_docs must be >= 1 with token offsets");
  if (cfg->dtype != MSA_F32 && cfg->dtype != MSA_BF16)
    return fail(MSA_ERR_INVALID_ARG, "dtype must be MSA_F32 or MSA_BF16");
  if (cfg->chunk_len < 2 || cfg->chunk_len > msa::kMaxChunkLen)
    return fail(MSA_ERR_UNSUPPORTED, "chunk_len=%d must be in [2, %d]", cfg->chunk_len,
                msa::kMaxChunkLen);
  if (cfg->head_dim != 64 && cfg->head_dim != 128)
    return fail(MSA_ERR_UNSUPPORTED, "head_dim=%d must be 64 or 128", cfg->head_dim);
  if (cfg->n_kv_heads < 1 || cfg->n_kv_heads * cfg->head_dim > 8192)
    return fail(MSA_ERR_UNSUPPORTED, "n_kv_heads=%d out of range", cfg->n_kv_heads);
  if (!pow2(cfg->router_dim) || cfg->router_dim < 16 || cfg->router_dim > 128)
    return fail(MSA_ERR_UNSUPPORTED, "router_dim=%d must be a power of two in [16, 128]",
                cfg->router_dim);
  const int W = cfg->n_router_heads * cfg->router_dim;
  if (cfg->n_router_heads < 1 || W % 64 != 0 || W > 4096)
    return fail(MSA_ERR_UNSUPPORTED,
                "n_router_heads * router_dim = %d must be a multiple of 64 and <= 4096", W);
  if (!(cfg->rope_theta > 1.0)) return fail(MSA_ERR_INVALID_ARG, "rope_theta must be > 1");
  if (cfg->max_local_position < 1)
    return fail(MSA_ERR_INVALID_ARG, "max_local_position must be >= 1");
  auto m = new msa_memory();
  m->n_docs = cfg->n_docs;
  m->chunk_len = cfg->chunk_len;
  m->H_kv = cfg->n_kv_heads;
  m->D = cfg->head_dim;
  m->H_r = cfg->n_router_heads;
  m->d_r = cfg->router_dim;
  m->dtype = cfg->dtype;
  m->theta = cfg->rope_theta;
  m->max_local_position = cfg->max_local_position;
  m->doc_tok_off.assign(cfg->doc_token_offsets, cfg->doc_token_offsets + cfg->n_docs + 1);
  m->doc_chunk_off.resize(cfg->n_docs + 1);
  if (m->doc_tok_off[0] != 0) {
    delete m;
    return fail(MSA_ERR_INVALID_ARG, "doc_token_offsets[0] must be 0");
  }
  m->doc_chunk_off[0] = 0;
  for (int d = 0; d < cfg->n_docs; ++d) {
    const int64_t len = m->doc_tok_off[d + 1] - m->doc_tok_off[d];
    if (len <= 0) {
      delete m;
      return fail(MSA_ERR_INVALID_ARG, "document %d is empty (offsets must increase)", d);
    }
    const int64_t nc = (len + m->chunk_len - 1) / m->chunk_len;
    m->doc_chunk_off[d + 1] = m->doc_chunk_off[d] + nc;
    m->max_doc_chunks = static_cast<int32_t>(std::max<int64_t>(m->max_doc_chunks, nc));
    m->max_doc_tokens = std::max<int64_t>(m->max_doc_tokens, len);
  }
  m->n_tokens = m->doc_tok_off[cfg->n_docs];
  m->n_chunks = m->doc_chunk_off[cfg->n_docs];
  if (m->n_chunks >= INT32_MAX) {
    delete m;
    return fail(MSA_ERR_UNSUPPORTED, "too many chunks");
  }
  m->rope_len = static_cast<int32_t>(
      std::max<int64_t>(m->max_doc_tokens, static_cast<int64_t>(m->max_local_position)));
  cudaGetDevice(&m->device);

  // host tables
  std::vector<int32_t> chunk_doc(m->n_chunks);
  for (int d = 0; d < cfg->n_docs; ++d)
    for (int64_t c = m->doc_chunk_off[d]; c < m->doc_chunk_off[d + 1]; ++c) chunk_doc[c] = d;
  const int half = m->D / 2;
  std::vector<float2> rope(static_cast<size_t>(m->rope_len) * half);
  for (int64_t p = 0; p < m->rope_len; ++p)
    for (int i = 0; i < half; ++i) {
      const double ang =
          static_cast<double>(p) * std::pow(m->theta, -2.0 * static_cast<double>(i) / m->D);
      rope[p * half + i] = make_float2(static_cast<float>(std::cos(ang)),
                                       static_cast<float>(std::sin(ang)));
    }
  auto alloc = [&](void **p, size_t n) { return cudaMalloc(p, std::max<size_t>(n, 16)); };
  if (alloc(reinterpret_cast<void **>(&m->d_chunk_doc), chunk_doc.size() * 4) != cudaSuccess ||
      alloc(reinterpret_cast<void **>(&m->d_doc_tok_off), m->doc_tok_off.size() * 8) != cudaSuccess ||
      alloc(reinterpret_cast<void **>(&m->d_doc_chunk_off), m->doc_chunk_off.size() * 8) != cudaSuccess ||
      alloc(reinterpret_cast<void **>(&m->d_rope), rope.size() * sizeof(float2)) != cudaSuccess) {
    cudaGetLastError();
    msa_memory_destroy(m);
    return fail(MSA_ERR_OUT_OF_MEMORY, "could not allocate the memory tables");
  }
  if (cudaMemcpy(m->d_chunk_doc, chunk_doc.data(), chunk_doc.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(m->d_doc_tok_off, m->doc_tok_off.data(), m->doc_tok_off.size() * 8, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(m->d_doc_chunk_off, m->doc_chunk_off.data(), m->doc_chunk_off.size() * 8, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(m->d_rope, rope.data(), rope.size() * sizeof(float2), cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaError_t e = cudaGetLastError();
    msa_memory_destroy(m);
    return cuda_fail(e, "uploading memory tables");
  }
  *out = m;
  return MSA_OK;
}

msa_status msa_memory_destroy(msa_memory *mem) {
  if (!mem) return fail(MSA_ERR_INVALID_ARG, "null memory");
  cudaFree(mem->d_chunk_doc);
  cudaFree(mem->d_doc_tok_off);
  cudaFree(mem->d_doc_chunk_off);
  cudaFree(mem->d_rope);
  delete mem;
  return MSA_OK;
}

msa_status msa_memory_get_info(const msa_memory *mem, msa_memory_info *out) {
  if (!mem || !out) return fail(MSA_ERR_INVALID_ARG, "null argument");
  const size_t es = elem_size(mem->dtype);
  out->n_tokens = mem->n_tokens;
  out->n_chunks = mem->n_chunks;
  out->max_doc_chunks = mem->max_doc_chunks;
  out->max_doc_tokens = mem->max_doc_tokens;
  out->elem_bytes = es;
  out->router_key_bytes = static_cast<size_t>(mem->n_chunks) * mem->H_r * mem->d_r * es;
  out->content_bytes = static_cast<size_t>(mem->n_chunks) * 2 * mem->H_kv * mem->D * es;
  out->doc_content_stride = static_cast<size_t>(mem->max_doc_chunks) * 2 * mem->H_kv * mem->D * es;
  return MSA_OK;
}

msa_status msa_memory_doc_chunk_offsets(const msa_memory *mem, int64_t *out) {
  if (!mem || !out) return fail(MSA_ERR_INVALID_ARG, "null argument");
  std::copy(mem->doc_chunk_off.begin(), mem->doc_chunk_off.end(), out);
  return MSA_OK;
}

msa_status msa_encode_memory(const msa_memory *mem, int32_t doc_begin, int32_t doc_count,
                             const void *K, const void *V, const void *Kr, void *router_keys,
                             void *content, void *router_mean, msa_stream stream) {
  if (!mem) return fail(MSA_ERR_INVALID_ARG, "null memory");
  if (doc_begin < 0 || doc_count < 1 || doc_count > mem->n_docs - doc_begin)
    return fail(MSA_ERR_INVALID_ARG, "document range [%d, %d+%d) outside [0, %d)", doc_begin,
                doc_begin, doc_count, mem->n_docs);
  if (!K || !V || !Kr || !router_keys || !content)
    return fail(MSA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(K) || !aligned16(V) || !aligned16(Kr) || !aligned16(router_keys) ||
      !aligned16(content) || !aligned16(router_mean))
    return fail(MSA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t c0 = mem->doc_chunk_off[doc_begin];
  const int64_t nc = mem->doc_chunk_off[doc_begin + doc_count] - c0;
  const int64_t tok_base = mem->doc_tok_off[doc_begin];
  if (nc > INT32_MAX) return fail(MSA_ERR_UNSUPPORTED, "too many chunks in one call");
  const int WK = mem->H_kv * mem->D, WR = mem->H_r * mem->d_r;
  const int thr_k = round32(WK / 8), thr_v = round32(WK / 4), thr_r = round32(WR / 4);
  if (thr_v > 1024 || thr_r > 1024) return fail(MSA_ERR_UNSUPPORTED, "rows too wide");
  const unsigned grid = static_cast<unsigned>(nc);
#define MSA_ENCODE(T)                                                                             \
  msa::pool_rope_kernel<T><<<grid, thr_k, 0, st>>>(                                               \
      static_cast<const T *>(K), tok_base, mem->H_kv, mem->D, c0, mem->d_chunk_doc,               \
      mem->d_doc_tok_off, mem->d_doc_chunk_off, mem->chunk_len, mem->d_rope,                      \
      static_cast<T *>(content), 2LL * WK);                                                       \
  MSA_LAUNCHED("pool_rope_kernel");                                                               \
  msa::pool_plain_kernel<T, false><<<grid, thr_v, 0, st>>>(                                       \
      static_cast<const T *>(V), tok_base, WK, c0, mem->d_chunk_doc, mem->d_doc_tok_off,          \
      mem->d_doc_chunk_off, mem->chunk_len, static_cast<T *>(content), 2LL * WK, WK, mem->D,      \
      nullptr);                                                                                   \
  MSA_LAUNCHED("pool_plain_kernel(V)");                                                           \
  msa::pool_plain_kernel<T, true><<<grid, thr_r, 0, st>>>(                                        \
      static_cast<const T *>(Kr), tok_base, WR, c0, mem->d_chunk_doc, mem->d_doc_tok_off,         \
      mem->d_doc_chunk_off, mem->chunk_len, static_cast<T *>(router_keys), WR, 0, mem->d_r,       \
      static_cast<T *>(router_mean));                                                             \
  MSA_LAUNCHED("pool_plain_kernel(Kr)");
  if (mem->dtype == MSA_BF16) {
    MSA_ENCODE(__nv_bfloat16)
  } else {
    MSA_ENCODE(float)
  }
#undef MSA_ENCODE
  return MSA_OK;
}

msa_status msa_route_reset(float *state, int64_t count, msa_stream stream) {
  if (!state || count < 1) return fail(MSA_ERR_INVALID_ARG, "null state or empty count");
  const int64_t blocks = std::min<int64_t>((count + 255) / 256, 4096);
  msa::fill_kernel<<<static_cast<unsigned>(blocks), 256, 0,
                     reinterpret_cast<cudaStream_t>(stream)>>>(state, count, -INFINITY);
  MSA_LAUNCHED("fill_kernel");
  return MSA_OK;
}

size_t msa_route_workspace_size(const msa_memory *mem, int32_t batch, int32_t tokens, int32_t k) {
  if (!mem || batch < 1 || tokens < 0 || k < 1) return 0;
  return plan_route(mem, batch, tokens, k).bytes;
}

msa_status msa_route(const msa_memory *mem, const void *router_keys, const void *Qr, int32_t batch,
                     int32_t tokens, int32_t k, const uint8_t *exclude, float *state, int32_t *ids,
                     float *scores, void *workspace, size_t workspace_bytes, msa_stream stream) {
  return route_impl(mem, router_keys, Qr, batch, tokens, k, exclude, state, ids, scores, workspace,
                    workspace_bytes, reinterpret_cast<cudaStream_t>(stream), 0, true);
}

size_t msa_attend_workspace_size(const msa_memory *mem, int32_t batch, int32_t tokens, int32_t k,
                                 int32_t n_q_heads) {
  if (!mem || batch < 1 || tokens < 1 || k < 0 || n_q_heads < 1) return 0;
  return plan_attend(mem, batch, tokens, k, n_q_heads, mem->max_local_position).bytes;
}

msa_status msa_sparse_attend(const msa_memory *mem, const void *content, const int32_t *ids,
                             int32_t batch, int32_t k, int32_t tokens, int32_t n_q_heads,
                             const void *Q, const void *K_new, const void *V_new, void *K_cache,
                             void *V_cache, int32_t *cache_len, int32_t cache_capacity,
                             int32_t pos_offset, void *O, void *workspace, size_t workspace_bytes,
                             msa_stream stream) {
  return attend_impl(mem, content, ids, nullptr, 0, batch, k, tokens, n_q_heads, Q, K_new, V_new,
                     K_cache, V_cache, cache_len, cache_capacity, pos_offset, O, workspace,
                     workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

msa_status msa_sparse_attend_static(const msa_memory *mem, const void *content,
                                    const int32_t *ids, int32_t batch, int32_t k, int32_t tokens,
                                    int32_t n_q_heads, const void *Q, const void *K_new,
                                    const void *V_new, void *K_cache, void *V_cache,
                                    int32_t *cache_len, int32_t cache_capacity,
                                    int32_t pos_offset, void *O, msa_stream stream) {
  const msa_status chk =
      attend_shape_check(mem, batch, k, tokens, n_q_heads, cache_capacity, pos_offset);
  if (chk != MSA_OK) return chk;
  const AttendPlan plan = plan_attend(mem, batch, tokens, k, n_q_heads, cache_capacity);
  if (plan.bytes > kStaticAttendScratchBytes)
    return fail(MSA_ERR_UNSUPPORTED,
                "this call needs %zu bytes of attention scratch; the static scratch holds %zu",
                plan.bytes, kStaticAttendScratchBytes);
  void *scratch = nullptr;
  const msa_status s = static_attend_scratch(&scratch);
  if (s != MSA_OK) return s;
  return attend_impl(mem, content, ids, nullptr, 0, batch, k, tokens, n_q_heads, Q, K_new, V_new,
                     K_cache, V_cache, cache_len, cache_capacity, pos_offset, O, scratch,
                     kStaticAttendScratchBytes, reinterpret_cast<cudaStream_t>(stream));
}

size_t msa_step_workspace_size(const msa_memory *mem, int32_t batch, int32_t k, int32_t n_q_heads) {
  if (!mem || batch < 1 || k < 1 || n_q_heads < 1) return 0;
  return round256(plan_route(mem, batch, 1, k).bytes) +
         plan_attend(mem, batch, 1, k, n_q_heads, mem->max_local_position).bytes;
}

msa_status msa_step(const msa_memory *mem, const void *router_keys, const void *content,
                    const msa_decode_state *s, const void *Qr_tok, const void *Q_tok,
                    const void *K_tok, const void *V_tok, void *O_tok, msa_stream stream) {
  if (!mem || !s) return fail(MSA_ERR_INVALID_ARG, "null memory or decode state");
  const size_t need = msa_step_workspace_size(mem, s->batch, s->top_k, s->n_q_heads);
  if (s->workspace_bytes < need || !s->workspace)
    return fail(MSA_ERR_INVALID_ARG, "decode workspace too small: %zu < %zu", s->workspace_bytes,
                need);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t route_bytes = round256(plan_route(mem, s->batch, 1, s->top_k).bytes);
  uint8_t *ws = static_cast<uint8_t *>(s->workspace);
  msa_status r = route_impl(mem, router_keys, Qr_tok, s->batch, 1, s->top_k, nullptr, s->state,
                            s->ids, s->scores, ws, route_bytes, st, 0, true);
  if (r != MSA_OK) return r;
  // the kernel before the attention is the route's top-k, which writes none of cache_len, the
  // token's Q/K/V or the local cache: the attention may start on its local part early
  return attend_impl(mem, content, s->ids, nullptr, 0, s->batch, s->top_k, 1, s->n_q_heads, Q_tok,
                     K_tok, V_tok, s->k_cache, s->v_cache, s->cache_len, s->cache_capacity,
                     s->pos_offset, O_tok, ws + route_bytes, s->workspace_bytes - route_bytes, st,
                     /*early=*/true);
}

msa_status msa_fetcher_create(const msa_memory *mem, const void *content_host, void *slot_cache,
                              int32_t n_slots, int32_t max_batch, int32_t max_k, uint32_t flags,
                              msa_fetcher **out) {
  if (!mem || !content_host || !slot_cache || !out)
    return fail(MSA_ERR_INVALID_ARG, "null argument");
  *out = nullptr;
  if (max_batch < 1 || max_k < 1 || max_k > msa::kMaxTopK)
    return fail(MSA_ERR_INVALID_ARG, "max_batch >= 1 and 1 <= max_k <= %d required", msa::kMaxTopK);
  if (static_cast<int64_t>(max_batch) * max_k > msa::kAssignMaxIds)
    return fail(MSA_ERR_UNSUPPORTED, "max_batch * max_k = %lld exceeds %d ids per fetch",
                (long long)max_batch * max_k, msa::kAssignMaxIds);
  if (static_cast<int64_t>(n_slots) < static_cast<int64_t>(max_batch) * max_k)
    return fail(MSA_ERR_INVALID_ARG, "n_slots=%d < max_batch * max_k = %lld", n_slots,
                (long long)max_batch * max_k);
  if (!aligned16(slot_cache)) return fail(MSA_ERR_INVALID_ARG, "slot cache must be 16-byte aligned");
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, content_host) != cudaSuccess ||
      attr.type != cudaMemoryTypeHost) {
    cudaGetLastError();
    return fail(MSA_ERR_INVALID_ARG, "content_host must be pinned (page-locked) host memory");
  }
  void *dev = nullptr;
  if (cudaHostGetDevicePointer(&dev, const_cast<void *>(content_host), 0) != cudaSuccess || !dev) {
    cudaGetLastError();
    return fail(MSA_ERR_UNSUPPORTED, "content_host is not mapped into the device address space");
  }
  auto f = new msa_fetcher();
  f->mem = mem;
  f->content_host = static_cast<const uint8_t *>(content_host);
  f->content_dev = static_cast<const uint8_t *>(dev);
  f->slot_cache = static_cast<uint8_t *>(slot_cache);
  f->n_slots = n_slots;
  f->max_batch = max_batch;
  f->max_k = max_k;
  f->flags = flags;
  f->row_bytes = static_cast<size_t>(2) * mem->H_kv * mem->D * elem_size(mem->dtype);
  f->slot_bytes = f->row_bytes * mem->max_doc_chunks;
  const size_t n = static_cast<size_t>(max_batch) * max_k;
  const size_t nd = static_cast<size_t>(mem->n_docs);
  auto dmalloc = [](void *p, size_t bytes) {
    return cudaMalloc(reinterpret_cast<void **>(p), bytes) == cudaSuccess;
  };
  bool ok = dmalloc(&f->d_doc_slot, nd * 4) && dmalloc(&f->d_claim, nd * 4) &&
            dmalloc(&f->d_slot_doc, static_cast<size_t>(n_slots) * 4) &&
            dmalloc(&f->d_slot_stamp, static_cast<size_t>(n_slots) * 4) &&
            dmalloc(&f->d_ctl, msa::kCtlN * 8) && dmalloc(&f->d_slots, n * 4) &&
            dmalloc(&f->d_list, n * 3 * 8) && dmalloc(&f->d_scratch, msa::kAssignScratch * 4) &&
            cudaEventCreateWithFlags(&f->ev_ids, cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&f->ev_fetch, cudaEventDisableTiming) == cudaSuccess;
  // bookkeeping: no document resident, no claim (any value above every index), stamps 0
  ok = ok && cudaMemset(f->d_doc_slot, 0xFF, nd * 4) == cudaSuccess &&
       cudaMemset(f->d_claim, 0x7F, nd * 4) == cudaSuccess &&
       cudaMemset(f->d_slot_doc, 0xFF, static_cast<size_t>(n_slots) * 4) == cudaSuccess &&
       cudaMemset(f->d_slot_stamp, 0, static_cast<size_t>(n_slots) * 4) == cudaSuccess &&
       cudaMemset(f->d_ctl, 0, msa::kCtlN * 8) == cudaSuccess &&
       cudaDeviceSynchronize() == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    msa_fetcher_destroy(f);
    return fail(MSA_ERR_OUT_OF_MEMORY, "could not allocate the fetcher's bookkeeping");
  }
  *out = f;
  return MSA_OK;
}

msa_status msa_fetcher_destroy(msa_fetcher *f) {
  if (!f) return fail(MSA_ERR_INVALID_ARG, "null fetcher");
  for (void *p : {static_cast<void *>(f->d_doc_slot), static_cast<void *>(f->d_claim),
                  static_cast<void *>(f->d_slot_doc), static_cast<void *>(f->d_slot_stamp),
                  static_cast<void *>(f->d_ctl), static_cast<void *>(f->d_slots),
                  static_cast<void *>(f->d_list), static_cast<void *>(f->d_scratch)})
    if (p) cudaFree(p);
  if (f->ev_ids) cudaEventDestroy(f->ev_ids);
  if (f->ev_fetch) cudaEventDestroy(f->ev_fetch);
  delete f;
  return MSA_OK;
}

msa_status msa_fetcher_stats(const msa_fetcher *f, int64_t *hits, int64_t *misses,
                             int64_t *copies, int64_t *bytes) {
  if (!f) return fail(MSA_ERR_INVALID_ARG, "null fetcher");
  int64_t ctl[msa::kCtlN];
  MSA_CUDA(cudaDeviceSynchronize());
  MSA_CUDA(cudaMemcpy(ctl, f->d_ctl, sizeof(ctl), cudaMemcpyDeviceToHost));
  if (hits) *hits = ctl[msa::kCtlHits];
  if (misses) *misses = ctl[msa::kCtlMisses];
  if (copies) *copies = ctl[msa::kCtlMisses];
  if (bytes) *bytes = ctl[msa::kCtlBytes];
  return MSA_OK;
}

msa_status msa_fetch(msa_fetcher *f, const int32_t *ids, int32_t batch, int32_t k,
                     msa_stream stream, msa_stream fetch_stream) {
  if (!f || !ids) return fail(MSA_ERR_INVALID_ARG, "null fetcher or ids");
  if (batch < 1 || batch > f->max_batch || k < 1 || k > f->max_k)
    return fail(MSA_ERR_INVALID_ARG, "batch=%d k=%d beyond the fetcher's %d x %d", batch, k,
                f->max_batch, f->max_k);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaStream_t fst = reinterpret_cast<cudaStream_t>(fetch_stream);
  const msa_memory *mem = f->mem;
  const int n = batch * k;
  // The fetch kernels prefer the largest shared-memory carveout (they use no shared memory):
  // an SM runs CTAs of one L1 / shared-memory split at a time, and the route kernel's split
  // is the largest, so with the same preference a fetch can run on the SMs beside it.
  static std::once_flag carveout;
  std::call_once(carveout, [] {
    cudaFuncSetAttribute(msa::fetch_assign_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                         cudaSharedmemCarveoutMaxShared);
    cudaFuncSetAttribute(msa::fetch_gather_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                         cudaSharedmemCarveoutMaxShared);
    cudaGetLastError();
  });
  // slot assignment after the top-k (stream order), then the copies on the fetch stream
  MSA_CUDA(launch_pdl(msa::fetch_assign_kernel, dim3(1), dim3(msa::kAssignThreads), 0, st, ids, n,
                      mem->n_docs, static_cast<const int64_t *>(mem->d_doc_chunk_off),
                      static_cast<int64_t>(f->row_bytes), static_cast<int64_t>(f->slot_bytes),
                      f->n_slots, (f->flags & MSA_FETCH_COLD) ? 1 : 0, f->d_doc_slot, f->d_claim,
                      f->d_slot_doc, f->d_slot_stamp, f->d_ctl, f->d_list, f->d_slots,
                      f->d_scratch));
  MSA_LAUNCHED("fetch_assign_kernel");
  if (fst != st) {
    MSA_CUDA(cudaEventRecord(f->ev_ids, st));
    MSA_CUDA(cudaStreamWaitEvent(fst, f->ev_ids, 0));
  }
  msa::fetch_gather_kernel<<<n, 256, 0, fst>>>(f->content_dev, f->slot_cache, f->d_list,
                                                f->d_ctl);
  MSA_LAUNCHED("fetch_gather_kernel");
  if (fst != st) {
    MSA_CUDA(cudaEventRecord(f->ev_fetch, fst));
    MSA_CUDA(cudaStreamWaitEvent(st, f->ev_fetch, 0));
  }
  return MSA_OK;
}

msa_status msa_sparse_attend_fetched(const msa_memory *mem, const msa_fetcher *f,
                                     const int32_t *ids, int32_t batch, int32_t k, int32_t tokens,
                                     int32_t n_q_heads, const void *Q, const void *K_new,
                                     const void *V_new, void *K_cache, void *V_cache,
                                     int32_t *cache_len, int32_t cache_capacity,
                                     int32_t pos_offset, void *O, void *workspace,
                                     size_t workspace_bytes, msa_stream stream) {
  if (!mem || !f) return fail(MSA_ERR_INVALID_ARG, "null memory or fetcher");
  if (f->mem != mem) return fail(MSA_ERR_INVALID_ARG, "fetcher belongs to another memory");
  if (batch > f->max_batch || k > f->max_k)
    return fail(MSA_ERR_INVALID_ARG, "batch / k beyond the fetcher's sizes");
  return attend_impl(mem, f->slot_cache, ids, f->d_slots, mem->max_doc_chunks, batch, k, tokens,
                     n_q_heads, Q, K_new, V_new, K_cache, V_cache, cache_len, cache_capacity,
                     pos_offset, O, workspace, workspace_bytes,
                     reinterpret_cast<cudaStream_t>(stream));
}

msa_status msa_step_host(const msa_memory *mem, const void *router_keys, msa_fetcher *f,
                         const msa_decode_state *s, const void *Qr_tok, const void *Q_tok,
                         const void *K_tok, const void *V_tok, void *O_tok, msa_stream stream,
                         msa_stream fetch_stream) {
  if (!mem || !s || !f) return fail(MSA_ERR_INVALID_ARG, "null memory, decode state or fetcher");
  const size_t need = msa_step_workspace_size(mem, s->batch, s->top_k, s->n_q_heads);
  if (s->workspace_bytes < need || !s->workspace)
    return fail(MSA_ERR_INVALID_ARG, "decode workspace too small: %zu < %zu", s->workspace_bytes,
                need);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t route_bytes = round256(plan_route(mem, s->batch, 1, s->top_k).bytes);
  uint8_t *ws = static_cast<uint8_t *>(s->workspace);
  msa_status r = route_impl(mem, router_keys, Qr_tok, s->batch, 1, s->top_k, nullptr, s->state,
                            s->ids, s->scores, ws, route_bytes, st, 0, true);
  if (r != MSA_OK) return r;
  r = msa_fetch(f, s->ids, s->batch, s->top_k, stream, fetch_stream);
  if (r != MSA_OK) return r;
  return attend_impl(mem, f->slot_cache, s->ids, f->d_slots, mem->max_doc_chunks, s->batch,
                     s->top_k, 1, s->n_q_heads, Q_tok, K_tok, V_tok, s->k_cache, s->v_cache,
                     s->cache_len, s->cache_capacity, s->pos_offset, O_tok, ws + route_bytes,
                     s->workspace_bytes - route_bytes, st);
}

// Workspace of msa_interleave(_adaptive): the route workspace for the largest
// round, the gathered rows [batch][k * max_doc_chunks][W], the per-query row
// counts, saved state rows [batch][n_docs] and the active flags [batch].
struct InterleavePlan {
  int cap = 0;
  size_t route = 0, rows = 0, count = 0, saved = 0, active = 0, bytes = 0;
};

InterleavePlan plan_interleave(const msa_memory *mem, int B, int T, int k) {
  InterleavePlan p;
  p.cap = k * mem->max_doc_chunks;
  const size_t W = static_cast<size_t>(mem->H_r) * mem->d_r;
  p.route = 0;
  const size_t rb = round256(plan_route(mem, B, std::max(T, p.cap), k).bytes);
  p.rows = rb;
  p.count = p.rows + round256(static_cast<size_t>(B) * p.cap * W * elem_size(mem->dtype));
  p.saved = p.count + round256(static_cast<size_t>(B) * 4);
  p.active = p.saved + round256(static_cast<size_t>(B) * mem->n_docs * 4);
  p.bytes = p.active + round256(static_cast<size_t>(B));
  return p;
}

size_t msa_interleave_workspace_size(const msa_memory *mem, int32_t batch, int32_t tokens,
                                     int32_t k) {
  if (!mem || batch < 1 || tokens < 1 || k < 1) return 0;
  return plan_interleave(mem, batch, tokens, k).bytes;
}

// Both interleave entry points: adaptive (n_rounds != nullptr) stops a query
// after the first round whose best new document scores below stop_score.
static msa_status interleave_impl(const msa_memory *mem, const void *router_keys, const void *Qr,
                           int32_t batch, int32_t tokens, int32_t k, int32_t rounds,
                           float stop_score, float *state, uint8_t *taken, int32_t *ids,
                           float *scores, int32_t *n_rounds, void *workspace,
                           size_t workspace_bytes, msa_stream stream) {
  if (!mem || !router_keys || !Qr || !state || !taken || !ids || !scores)
    return fail(MSA_ERR_INVALID_ARG, "null argument");
  if (batch < 1 || tokens < 1 || rounds < 1 || k < 1 || k > mem->n_docs || k > msa::kMaxTopK)
    return fail(MSA_ERR_INVALID_ARG, "bad batch, tokens, rounds or k");
  const InterleavePlan plan = plan_interleave(mem, batch, tokens, k);
  if (!workspace || workspace_bytes < plan.bytes)
    return fail(MSA_ERR_INVALID_ARG, "workspace too small: %zu < %zu", workspace_bytes, plan.bytes);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  void *rows = ws + plan.rows;
  int32_t *count = reinterpret_cast<int32_t *>(ws + plan.count);
  float *saved = reinterpret_cast<float *>(ws + plan.saved);
  uint8_t *active = ws + plan.active;
  const int W = mem->H_r * mem->d_r;
  const int64_t nd = static_cast<int64_t>(batch) * mem->n_docs;
  msa_status r = msa_route_reset(state, nd, stream);
  if (r != MSA_OK) return r;
  MSA_CUDA(cudaMemsetAsync(taken, 0, static_cast<size_t>(nd), st));
  if (n_rounds) {
    MSA_CUDA(cudaMemsetAsync(active, 1, static_cast<size_t>(batch), st));
    MSA_CUDA(cudaMemsetAsync(n_rounds, 0, static_cast<size_t>(batch) * sizeof(int32_t), st));
  }
  const void *q = Qr;
  int T = tokens;
  bool hold = false;  // some query has no new rows this round
  std::vector<int32_t> h_count(batch);
  for (int round = 0; round < rounds; ++round) {
    int32_t *ids_r = ids + static_cast<int64_t>(round) * batch * k;
    float *sc_r = scores + static_cast<int64_t>(round) * batch * k;
    if (hold) {
      msa::hold_state_kernel<<<batch, 256, 0, st>>>(state, saved, count, mem->n_docs, 0);
      MSA_LAUNCHED("hold_state_kernel");
    }
    r = route_impl(mem, router_keys, q, batch, T, k, taken, state, ids_r, sc_r, ws, plan.rows, st,
                   q == Qr ? T : plan.cap, q == Qr);
    if (r != MSA_OK) return r;
    if (hold) {
      msa::hold_state_kernel<<<batch, 256, 0, st>>>(state, saved, count, mem->n_docs, 1);
      MSA_LAUNCHED("hold_state_kernel");
    }
    if (n_rounds) {
      msa::interleave_stop_kernel<<<(batch + 127) / 128, 128, 0, st>>>(
          ids_r, sc_r, batch, k, stop_score, active, n_rounds, round);
      MSA_LAUNCHED("interleave_stop_kernel");
    }
    if (round + 1 == rounds) break;
    if (mem->dtype == MSA_BF16) {
      msa::gather_rows_kernel<__nv_bfloat16><<<batch, 256, 0, st>>>(
          static_cast<const __nv_bfloat16 *>(router_keys), ids_r, k, mem->d_doc_chunk_off,
          mem->n_docs, W, static_cast<__nv_bfloat16 *>(rows), plan.cap, taken, count);
    } else {
      msa::gather_rows_kernel<float><<<batch, 256, 0, st>>>(
          static_cast<const float *>(router_keys), ids_r, k, mem->d_doc_chunk_off, mem->n_docs, W,
          static_cast<float *>(rows), plan.cap, taken, count);
    }
    MSA_LAUNCHED("gather_rows_kernel");
    MSA_CUDA(cudaMemcpyAsync(h_count.data(), count, batch * sizeof(int32_t),
                             cudaMemcpyDeviceToHost, st));
    MSA_CUDA(cudaStreamSynchronize(st));
    int T_next = 0;
    hold = false;
    for (int b = 0; b < batch; ++b) {
      T_next = std::max(T_next, static_cast<int>(h_count[b]));
      hold = hold || h_count[b] == 0;
    }
    if (T_next == 0) {
      // no query has new rows: the remaining rounds retrieve nothing
      for (int rr = round + 1; rr < rounds; ++rr) {
        MSA_CUDA(cudaMemsetAsync(ids + static_cast<int64_t>(rr) * batch * k, 0xFF,
                                 static_cast<size_t>(batch) * k * sizeof(int32_t), st));
        const int64_t n = static_cast<int64_t>(batch) * k;
        msa::fill_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(
            scores + static_cast<int64_t>(rr) * batch * k, n, -INFINITY);
        MSA_LAUNCHED("fill_kernel");
      }
      break;
    }
    if (mem->dtype == MSA_BF16) {
      msa::pad_rows_kernel<__nv_bfloat16><<<batch, 256, 0, st>>>(
          static_cast<__nv_bfloat16 *>(rows), plan.cap, W, count, T_next);
    } else {
      msa::pad_rows_kernel<float><<<batch, 256, 0, st>>>(static_cast<float *>(rows), plan.cap, W,
                                                          count, T_next);
    }
    MSA_LAUNCHED("pad_rows_kernel");
    // rows[b] holds cap rows; the route reads the first T_next of each (row pitch cap)
    q = rows;
    T = T_next;
  }
  return MSA_OK;
}

msa_status msa_interleave(const msa_memory *mem, const void *router_keys, const void *Qr,
                          int32_t batch, int32_t tokens, int32_t k, int32_t rounds, float *state,
                          uint8_t *taken, int32_t *ids, float *scores, void *workspace,
                          size_t workspace_bytes, msa_stream stream) {
  return interleave_impl(mem, router_keys, Qr, batch, tokens, k, rounds, -INFINITY, state, taken,
                         ids, scores, nullptr, workspace, workspace_bytes, stream);
}

msa_status msa_interleave_adaptive(const msa_memory *mem, const void *router_keys,
                                   const void *Qr, int32_t batch, int32_t tokens, int32_t k,
                                   int32_t max_rounds, float stop_score, float *state,
                                   uint8_t *taken, int32_t *ids, float *scores,
                                   int32_t *n_rounds, void *workspace, size_t workspace_bytes,
                                   msa_stream stream) {
  if (!n_rounds) return fail(MSA_ERR_INVALID_ARG, "null n_rounds");
  if (stop_score != stop_score) return fail(MSA_ERR_INVALID_ARG, "stop_score is NaN");
  return interleave_impl(mem, router_keys, Qr, batch, tokens, k, max_rounds, stop_score, state,
                         taken, ids, scores, n_rounds, workspace, workspace_bytes, stream);
}

msa_status msa_topk_merge(const float *cand_scores, const int32_t *cand_ids, int32_t n_shards,
                          int32_t batch, int32_t k_cand, const int32_t *shard_doc_base, int32_t k,
                          int32_t *ids, float *scores, msa_stream stream) {
  if (!cand_scores || !cand_ids || !shard_doc_base || !ids || !scores)
    return fail(MSA_ERR_INVALID_ARG, "null argument");
  if (n_shards < 1 || n_shards > msa::kMaxShards)
    return fail(MSA_ERR_INVALID_ARG, "n_shards=%d must be in [1, %d]", n_shards, msa::kMaxShards);
  if (k_cand < 1 || k_cand > msa::kMaxTopK)
    return fail(MSA_ERR_INVALID_ARG, "k_cand=%d must be in [1, %d]", k_cand, msa::kMaxTopK);
  if (static_cast<int64_t>(n_shards) * k_cand > msa::kTopkSlice)
    return fail(MSA_ERR_UNSUPPORTED, "n_shards * k_cand = %d exceeds %d candidates",
                n_shards * k_cand, msa::kTopkSlice);
  if (k < 1 || k > msa::kMaxTopK || k > n_shards * k_cand)
    return fail(MSA_ERR_INVALID_ARG, "k=%d must be in [1, min(%d, n_shards * k_cand)]", k,
                msa::kMaxTopK);
  if (batch < 1 || batch > 65535) return fail(MSA_ERR_INVALID_ARG, "batch=%d out of range", batch);
  msa::ShardBases bases = {};
  for (int s = 0; s < n_shards; ++s) {
    if (shard_doc_base[s] < 0 || (s > 0 && shard_doc_base[s] < shard_doc_base[s - 1]))
      return fail(MSA_ERR_INVALID_ARG, "shard_doc_base must be non-negative and non-decreasing");
    bases.base[s] = shard_doc_base[s];
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#define MSA_MERGE(KL)                                                                           \
  MSA_CUDA(launch_pdl(msa::topk_merge_shards_kernel<KL>, dim3(batch), dim3(msa::kTopkThreads), \
                      0, st, cand_scores, cand_ids, n_shards, batch, k_cand, bases, k, ids,     \
                      scores));
  if (k <= 16) {
    MSA_MERGE(16)
  } else if (k <= 32) {
    MSA_MERGE(32)
  } else {
    MSA_MERGE(64)
  }
#undef MSA_MERGE
  MSA_LAUNCHED("topk_merge_shards_kernel");
  return MSA_OK;
}

msa_status msa_route_backward(const msa_memory *mem, const void *router_mean, const void *Qr,
                              int32_t batch, int32_t tokens, const float *d_score, float *d_Qr,
                              float *d_router_mean, msa_stream stream) {
  if (!mem || !router_mean || !Qr || !d_score || !d_Qr || !d_router_mean)
    return fail(MSA_ERR_INVALID_ARG, "null argument");
  if (batch < 1 || tokens < 1) return fail(MSA_ERR_INVALID_ARG, "batch and tokens must be >= 1");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t W = static_cast<int64_t>(mem->H_r) * mem->d_r;
  MSA_CUDA(cudaMemsetAsync(d_Qr, 0, static_cast<size_t>(batch) * tokens * W * 4, st));
  MSA_CUDA(cudaMemsetAsync(d_router_mean, 0, static_cast<size_t>(mem->n_chunks) * W * 4, st));
  const int64_t warps = static_cast<int64_t>(batch) * mem->n_docs;
  const unsigned grid =
      static_cast<unsigned>(std::min<int64_t>((warps + 7) / 8, static_cast<int64_t>(num_sms()) * 8));
  if (mem->dtype == MSA_BF16)
    msa::route_backward_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        static_cast<const __nv_bfloat16 *>(Qr), batch, tokens,
        static_cast<const __nv_bfloat16 *>(router_mean), mem->d_doc_chunk_off, mem->n_docs,
        mem->H_r, mem->d_r, d_score, d_Qr, d_router_mean);
  else
    msa::route_backward_kernel<float><<<grid, 256, 0, st>>>(
        static_cast<const float *>(Qr), batch, tokens, static_cast<const float *>(router_mean),
        mem->d_doc_chunk_off, mem->n_docs, mem->H_r, mem->d_r, d_score, d_Qr, d_router_mean);
  MSA_LAUNCHED("route_backward_kernel");
  return MSA_OK;
}

msa_status msa_sparse_attend_backward(const msa_memory *mem, const void *content,
                                      const int32_t *ids, int32_t batch, int32_t k,
                                      int32_t tokens, int32_t n_q_heads, const void *Q,
                                      const void *K_cache, const void *V_cache,
                                      const int32_t *cache_len0, int32_t cache_capacity,
                                      int32_t pos_offset, const void *dO, float *dQ,
                                      float *d_cache_k, float *d_cache_v, float *d_content,
                                      msa_stream stream) {
  const msa_status chk =
      attend_shape_check(mem, batch, k, tokens, n_q_heads, cache_capacity, pos_offset);
  if (chk != MSA_OK) return chk;
  if (n_q_heads > 32)
    return fail(MSA_ERR_UNSUPPORTED, "the attention backward takes at most 32 query heads");
  if (!content || (k > 0 && !ids) || !Q || !K_cache || !V_cache || !cache_len0 || !dO || !dQ ||
      !d_cache_k || !d_cache_v || !d_content)
    return fail(MSA_ERR_INVALID_ARG, "null pointer argument");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t row = static_cast<size_t>(mem->H_kv) * mem->D * 4;
  MSA_CUDA(cudaMemsetAsync(d_content, 0, static_cast<size_t>(mem->n_chunks) * 2 * row, st));
  MSA_CUDA(cudaMemsetAsync(d_cache_k, 0, static_cast<size_t>(batch) * cache_capacity * row, st));
  MSA_CUDA(cudaMemsetAsync(d_cache_v, 0, static_cast<size_t>(batch) * cache_capacity * row, st));
  const float scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(mem->D)));
  const dim3 grid(static_cast<unsigned>(static_cast<int64_t>(batch) * tokens));
  const dim3 block(static_cast<unsigned>(n_q_heads * 32));
#define MSA_ATT_BWD(T, DD)                                                                          \
  msa::attend_backward_kernel<T, DD><<<grid, block, 0, st>>>(                                      \
      static_cast<const T *>(content), ids, k, mem->d_doc_chunk_off, mem->n_docs, mem->H_kv,      \
      n_q_heads, static_cast<const T *>(Q), tokens, static_cast<const T *>(K_cache),              \
      static_cast<const T *>(V_cache), cache_len0, cache_capacity, pos_offset, mem->d_rope, scale, \
      static_cast<const T *>(dO), dQ, d_content, d_cache_k, d_cache_v);
  if (mem->dtype == MSA_BF16) {
    if (mem->D == 128) { MSA_ATT_BWD(__nv_bfloat16, 128) } else { MSA_ATT_BWD(__nv_bfloat16, 64) }
  } else {
    if (mem->D == 128) { MSA_ATT_BWD(float, 128) } else { MSA_ATT_BWD(float, 64) }
  }
#undef MSA_ATT_BWD
  MSA_LAUNCHED("attend_backward_kernel");
  return MSA_OK;
}

msa_status msa_device_error(uint32_t *bits, msa_stream stream) {
  if (!bits) return fail(MSA_ERR_INVALID_ARG, "null output");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned int v = 0, zero = 0;
  MSA_CUDA(cudaMemcpyFromSymbolAsync(&v, msa::g_device_error, sizeof(v), 0,
                                     cudaMemcpyDeviceToHost, st));
  MSA_CUDA(cudaMemcpyToSymbolAsync(msa::g_device_error, &zero, sizeof(zero), 0,
                                   cudaMemcpyHostToDevice, st));
  MSA_CUDA(cudaStreamSynchronize(st));
  *bits = v;
  if (v & MSA_DEVERR_WAIT_TIMEOUT) return fail(MSA_ERR_TIMEOUT, "a device wait timed out");
  if (v) return fail(MSA_ERR_STATE, "device bounds check fired (bits 0x%x)", v);
  return MSA_OK;
}

}  // extern "C"
