// Host side of the C ABI declared in include/sd_api.h: argument checks,
// workspace carve-up, kernel selection and launches on the caller's stream.
// Nothing here allocates or synchronises (except sd_get_device_errors).

#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <stdint.h>

#include "../../include/sd_api.h"
#include "attn_mma.cuh"
#include "attn_umma.cuh"
#include "indexer_dp4a.cuh"
#include "indexer_umma.cuh"
#include "sd_common.cuh"
#include "sparse_index.cuh"
#include "topk_cluster.cuh"
#include "topk_radix.cuh"
#include "triattention.cuh"

namespace {

thread_local int32_t t_last_cuda_error = 0;
thread_local int32_t t_launches = 0;
thread_local cudaEvent_t t_stage_events[8];
thread_local int32_t t_stage_count = 0;

enum Stage { kStageIndexer = 0, kStageTopk = 1, kStageAttn = 2, kStageCombine = 3 };

void stage_mark(int stage, int edge, cudaStream_t st) {
  // external: inside a stream capture the record becomes a real event node that
  // a host can time after each graph replay
  if (stage < t_stage_count) cudaEventRecordWithFlags(t_stage_events[2 * stage + edge], st, cudaEventRecordExternal);
}

// Polls the eviction compaction's cross-CTA waits make before giving up
// (sd_set_wait_limit; a launch argument, read on the host at launch).
std::atomic<uint32_t> g_tri_wait_limit{sd::kTriWaitLimit};

constexpr size_t kAlign = 256;
constexpr int kMaxK = 2048;
constexpr int kMaxSeqlen = 1 << 20;
constexpr int kAttnTargetCtas = 296;  // two waves' worth of CTAs on 148 SMs
constexpr int kAttnMaxSplits = 16;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

sd_status cuda_check(cudaError_t e) {
  if (e == cudaSuccess) return SD_OK;
  t_last_cuda_error = static_cast<int32_t>(e);
  return SD_ERR_CUDA;
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (device, kernel,
// size): the attribute outlives the call, and setting it on every launch
// costs host time on the decode loop.
sd_status set_smem_limit(const void* kern, size_t bytes) {
  struct Entry { const void* k; int dev; size_t bytes; };
  static std::mutex mu;
  static Entry done[64];
  static int n_done = 0;
  int dev = 0;
  sd_status s = cuda_check(cudaGetDevice(&dev));
  if (s != SD_OK) return s;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n_done; ++i)
    if (done[i].k == kern && done[i].dev == dev && done[i].bytes >= bytes) return SD_OK;
  s = cuda_check(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)));
  if (s != SD_OK) return s;
  for (int i = 0; i < n_done; ++i)
    if (done[i].k == kern && done[i].dev == dev) {
      done[i].bytes = bytes;
      return SD_OK;
    }
  if (n_done < 64) done[n_done++] = Entry{kern, dev, bytes};
  return SD_OK;
}

sd_status after_launch() {
  ++t_launches;
  return cuda_check(cudaGetLastError());
}

// Launches a kernel with programmatic dependent launch allowed, so that its
// launch and set-up overlap the tail of the previous kernel in the stream
// (every kernel of this library waits in pdl_wait() before reading earlier
// results). Off while stage events are armed: an event between two kernels
// must see the first one complete.
template <typename... KArgs, typename... Args>
sd_status launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = t_stage_count == 0 ? 1 : 0;
  ++t_launches;
  return cuda_check(cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...));
}

struct AttnPlan {
  int mt, hb, n_hb, n_splits, slots_per_split;
};

// Split plan for the attention: a deterministic function of the shape only,
// so that sd_workspace_size() can size the partials without a device query.
AttnPlan attn_plan(int B, int G, int H, int k) {
  AttnPlan p;
  const int qpk = H / G;
  p.mt = qpk >= 32 ? 2 : 1;
  p.hb = 16 * p.mt;
  p.n_hb = sd::ceil_div(qpk, p.hb);
  const long long base = (long long)B * G * p.n_hb;
  const int max_splits = std::min(kAttnMaxSplits, sd::ceil_div(k, sd::kAttnTile));
  long long want = (kAttnTargetCtas + base - 1) / base;
  int splits = static_cast<int>(std::max(1LL, std::min<long long>(want, max_splits)));
  p.slots_per_split = sd::ceil_div(sd::ceil_div(k, splits), sd::kAttnTile) * sd::kAttnTile;
  p.n_splits = sd::ceil_div(k, p.slots_per_split);
  return p;
}

size_t scores_bytes(int B, int G, int max_seqlen) {
  return align_up(sizeof(int32_t) * (size_t)B * G * (size_t)max_seqlen);
}

// The tensor-core MLA attention serves the 128-head, 576/512 latent-row shape.
bool umma_attn_fits(int G, int H, int Dk, int Dv, bool v_separate) {
  return !v_separate && G == 1 && H == sd::kAuHeads && Dk == sd::kAuDk && Dv == sd::kAuDv;
}

size_t attn_bytes(int B, int G, int H, int k, int Dv) {
  const AttnPlan p = attn_plan(B, G, H, k);
  const size_t n = (size_t)B * H * p.n_splits;
  size_t bytes = align_up(sizeof(float) * n * Dv) + align_up(sizeof(float2) * n);
  if (G == 1 && H == sd::kAuHeads && Dv == sd::kAuDv) bytes = std::max(bytes, align_up(sd::attn_umma_workspace(B, k)));
  return bytes;
}

bool ws_ok(const void* ws, size_t have, size_t need) {
  if (need == 0) return true;
  return ws != nullptr && have >= need && (reinterpret_cast<uintptr_t>(ws) % kAlign) == 0;
}

bool geom_ok(const sd_paged_desc& pd) {
  return pd.num_pages > 0 && pd.page_size > 0 && pd.max_pages_per_req > 0 && pd.kv_heads > 0;
}

sd_status check_indexer_args(const int8_t* qi, const int32_t* w, const int8_t* ki_pages,
                             const int32_t* bt, const int32_t* seqlens, const sd_paged_desc& pd,
                             int B, int Hi, int Di, int max_seqlen, int k, const int32_t* indices) {
  if (!qi || !w || !ki_pages || !bt || !seqlens || !indices) return SD_ERR_INVALID_ARG;
  if (!geom_ok(pd) || B < 0 || Hi <= 0 || Di <= 0 || max_seqlen < 0 || k <= 0)
    return SD_ERR_INVALID_ARG;
  if (Di != 32 && Di != 64 && Di != 128) return SD_ERR_UNSUPPORTED;
  if (Hi > 64 || pd.kv_heads * Di > 1024) return SD_ERR_UNSUPPORTED;
  // key rows are copied in 16-byte units (bulk copies, TMA)
  if ((reinterpret_cast<uintptr_t>(ki_pages) & 15u) != 0) return SD_ERR_INVALID_ARG;
  if (k > kMaxK || max_seqlen > kMaxSeqlen) return SD_ERR_UNSUPPORTED;
  return SD_OK;
}

sd_status check_attn_args(const uint16_t* q, const uint16_t* k_pages, const int32_t* bt,
                          const int32_t* seqlens, const int32_t* indices, const sd_paged_desc& pd,
                          int B, int H, int Dk, int Dv, int k, float scale, const uint16_t* out,
                          bool v_separate) {
  if (!q || !k_pages || !bt || !seqlens || !indices || !out) return SD_ERR_INVALID_ARG;
  if (!geom_ok(pd) || B < 0 || H <= 0 || Dk <= 0 || Dv <= 0 || k <= 0 || !isfinite(scale))
    return SD_ERR_INVALID_ARG;
  if (H % pd.kv_heads != 0) return SD_ERR_INVALID_ARG;
  if (!v_separate && Dv > Dk) return SD_ERR_INVALID_ARG;
  const bool shape_ok = (Dk == 64 && Dv == 64) || (Dk == 128 && Dv == 128) || (Dk == 576 && Dv == 512);
  if (!shape_ok || H / pd.kv_heads > 128 || k > kMaxK) return SD_ERR_UNSUPPORTED;
  return SD_OK;
}

template <int DI>
sd_status launch_indexer_t(const int8_t* qi, const int32_t* w, const int8_t* ki, const int32_t* bt,
                           const int32_t* seqlens, int32_t* scores, const sd_paged_desc& pd, int B,
                           int Hi, int max_seqlen, cudaStream_t st) {
  const size_t smem = sd::indexer_dp4a_smem(pd.kv_heads, Hi, DI);
  if (smem > 48 * 1024) {
    const sd_status s = set_smem_limit(reinterpret_cast<const void*>(sd::indexer_dp4a_kernel<DI>), smem);
    if (s != SD_OK) return s;
  }
  dim3 grid(sd::ceil_div(max_seqlen, sd::indexer_dp4a_tokens(pd.kv_heads, DI)), B);
  stage_mark(kStageIndexer, 0, st);
  const sd_status s = launch_k(sd::indexer_dp4a_kernel<DI>, grid, dim3(sd::kIdxThreads), smem, st, qi, w, ki, bt,
                               seqlens, scores, pd.num_pages, pd.page_size, pd.max_pages_per_req, pd.kv_heads, Hi,
                               max_seqlen);
  stage_mark(kStageIndexer, 1, st);
  return s;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// dependency on libcuda); looked up once per process.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// A 2-D int8 map over `rows` rows of row_bytes bytes, boxes of box_rows x 128 B
// (one 128-byte column chunk), 128-byte swizzle (the K-major UMMA operand
// layout).
bool encode_rows128(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows, uint64_t row_bytes = 128) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (fn == nullptr || (reinterpret_cast<uintptr_t>(base) & 15u) != 0) return false;
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estride[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A 2-D bf16 map (row-major, `row_bytes` apart) with boxes of box_cols x box_rows
// and 128-byte swizzle; box_cols * 2 must be 128.
bool encode_bf16_rows(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                      uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (fn == nullptr || (reinterpret_cast<uintptr_t>(base) & 15u) != 0 || (row_bytes & 15u) != 0) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estride[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 148;
  return n;
}

// The tensor-core indexer covers one KV head of 128-byte keys with 64 heads
// (MLA) and 8 KV heads of 64-byte keys with 4 heads each (per-head
// selection), with pages that tile a 128-token block; everything else takes
// the dp4a kernel.
bool umma_indexer_mla(const sd_paged_desc& pd, int Hi, int Di) { return pd.kv_heads == 1 && Di == 128 && Hi == 64; }
bool umma_indexer_perhead(const sd_paged_desc& pd, int Hi, int Di) { return pd.kv_heads == 8 && Di == 64 && Hi == 4; }
bool umma_indexer_fits(const sd_paged_desc& pd, int Hi, int Di, const void* qi, const void* ki) {
  const int P = pd.page_size;
  return (umma_indexer_mla(pd, Hi, Di) || umma_indexer_perhead(pd, Hi, Di)) && P >= 8 && P <= 128 && (128 % P) == 0 &&
         (long long)(pd.num_pages + 1) * P < (1ll << 31) &&  // TMA row coordinates, one page past the end included
         (reinterpret_cast<uintptr_t>(qi) & 15u) == 0 && (reinterpret_cast<uintptr_t>(ki) & 15u) == 0;
}

template <class Cfg, int G, int HPG, int DI>
sd_status launch_indexer_umma_t(const int8_t* qi, const int32_t* w, const int8_t* ki, const int32_t* bt,
                                const int32_t* seqlens, int32_t* scores, const sd_paged_desc& pd, int B,
                                int max_seqlen, cudaStream_t st, bool* launched) {
  *launched = false;
  CUtensorMap tm_keys, tm_q;
  if (!encode_rows128(&tm_keys, ki, (uint64_t)pd.num_pages * pd.page_size, pd.page_size, (uint64_t)G * DI)) return SD_OK;
  if (G == 1) {
    if (!encode_rows128(&tm_q, qi, (uint64_t)B * Cfg::kHeads, Cfg::kHeads)) return SD_OK;
  } else {
    tm_q = tm_keys;  // unused: the block-diagonal query operand is built in shared memory
  }
  auto kern = sd::indexer_umma_kernel<Cfg, G, HPG, DI>;
  sd_status s = set_smem_limit(reinterpret_cast<const void*>(kern), Cfg::kSmemAlloc);
  if (s != SD_OK) return s;
  stage_mark(kStageIndexer, 0, st);
  s = launch_k(kern, dim3(sm_count()), dim3(sd::kUmmaThreads), Cfg::kSmemAlloc, st, tm_keys, tm_q, qi, w, bt,
               seqlens, scores, B, pd.num_pages, pd.page_size, pd.max_pages_per_req, max_seqlen);
  stage_mark(kStageIndexer, 1, st);
  *launched = true;
  return s;
}

sd_status launch_indexer_umma(const int8_t* qi, const int32_t* w, const int8_t* ki, const int32_t* bt,
                              const int32_t* seqlens, int32_t* scores, const sd_paged_desc& pd, int B, int Hi,
                              int Di, int max_seqlen, cudaStream_t st, bool* launched) {
  if (umma_indexer_mla(pd, Hi, Di))
    return launch_indexer_umma_t<sd::IdxCfgMla, 1, 64, 128>(qi, w, ki, bt, seqlens, scores, pd, B, max_seqlen, st,
                                                           launched);
  return launch_indexer_umma_t<sd::IdxCfgPerHead, 8, 4, 64>(qi, w, ki, bt, seqlens, scores, pd, B, max_seqlen, st,
                                                           launched);
}

template <int PER, int NT>
sd_status launch_topk_cluster(const int32_t* scores, const int32_t* seqlens, int32_t* indices, int rows, int G,
                              int max_seqlen, int cap, int k, int cs, const sd::RowMap& rm, const int32_t* hint,
                              cudaStream_t st) {
  const size_t smem = sizeof(sd::TopkClusterSmem<PER, NT>);
  sd_status s = set_smem_limit(reinterpret_cast<const void*>(sd::topk_cluster_kernel<PER, NT>), smem);
  if (s != SD_OK) return s;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, rows, 1);
  cfg.blockDim = dim3(NT, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = t_stage_count == 0 ? 2 : 1;  // see launch_k
  return cuda_check(cudaLaunchKernelEx(&cfg, sd::topk_cluster_kernel<PER, NT>, scores, seqlens, indices, G,
                                       std::max(max_seqlen, 1), cap, k, rm, hint));
}

// Top-k: one thread-block cluster per row when the row fits in the cluster's
// shared memory (max_seqlen <= 8 x 1024 x 32), else one CTA per row over L2.
sd_status launch_topk(const int32_t* scores, const int32_t* seqlens, int32_t* indices, int B, int G,
                      int max_seqlen, int cap, int k, const sd::RowMap& rm, const int32_t* hint, cudaStream_t st) {
  const int rows = B * G;
  const long long sms = sm_count();
  const int cs16 = sd::topk_cluster_size(max_seqlen, 16, 1024);   // 1024 threads, one CTA per SM
  const int cs32 = sd::topk_cluster_size(max_seqlen, 32, 1024);
  const int cs32h = sd::topk_cluster_size(max_seqlen, 32, 512);   // 512 threads, two CTAs per SM
  stage_mark(kStageTopk, 0, st);
  if ((cs16 > 0 || cs32 > 0) && rows <= 65535) {
    // All rows' CTAs in one wave if possible: 1024 threads x 16 scores (the
    // most warps per row) when a CTA per SM is enough, else 512 x 32 when two
    // per SM are, else 1024 x 32 (the fewest CTAs)
    sd_status s;
    if (cs16 > 0 && (long long)rows * cs16 <= sms)
      s = launch_topk_cluster<16, 1024>(scores, seqlens, indices, rows, G, max_seqlen, cap, k, cs16, rm, hint, st);
    else if (cs32h > 0 && (long long)rows * cs32h <= 2 * sms)
      s = launch_topk_cluster<32, 512>(scores, seqlens, indices, rows, G, max_seqlen, cap, k, cs32h, rm, hint, st);
    else  // cs32 > 0 here: a row that fits at 16 scores per thread fits at 32
      s = launch_topk_cluster<32, 1024>(scores, seqlens, indices, rows, G, max_seqlen, cap, k, cs32, rm, hint, st);
    stage_mark(kStageTopk, 1, st);
    ++t_launches;
    return s;
  }
  const sd_status s = launch_k(sd::topk_radix_kernel, dim3(rows), dim3(sd::kTopkThreads), 0, st, scores, seqlens,
                               indices, G, std::max(max_seqlen, 1), cap, k, rm);
  stage_mark(kStageTopk, 1, st);
  return s;
}

sd_status launch_indexer_topk(const int8_t* qi, const int32_t* w, const int8_t* ki, const int32_t* bt,
                              const int32_t* seqlens, const sd_paged_desc& pd, int B, int Hi, int Di,
                              int max_seqlen, int k, int32_t* indices, int32_t* scores,
                              cudaStream_t st, const sd::RowMap& rm = sd::RowMap{}, const int32_t* hint = nullptr) {
  const int G = pd.kv_heads;
  if (B == 0) return SD_OK;
  bool done = false;
  if (max_seqlen > 0 && umma_indexer_fits(pd, Hi, Di, qi, ki)) {
    sd_status s = launch_indexer_umma(qi, w, ki, bt, seqlens, scores, pd, B, Hi, Di, max_seqlen, st, &done);
    if (s != SD_OK) return s;
  }
  if (max_seqlen > 0 && !done) {
    sd_status s = SD_OK;
    if (Di == 32) s = launch_indexer_t<32>(qi, w, ki, bt, seqlens, scores, pd, B, Hi, max_seqlen, st);
    else if (Di == 64) s = launch_indexer_t<64>(qi, w, ki, bt, seqlens, scores, pd, B, Hi, max_seqlen, st);
    else s = launch_indexer_t<128>(qi, w, ki, bt, seqlens, scores, pd, B, Hi, max_seqlen, st);
    if (s != SD_OK) return s;
  }
  const int cap = std::min(max_seqlen, pd.max_pages_per_req * pd.page_size);
  return launch_topk(scores, seqlens, indices, B, G, max_seqlen, cap, k, rm, hint, st);
}

template <int DK, int DV, int MT>
sd_status launch_attn_t(const uint16_t* q, const uint16_t* kp, const uint16_t* vp, const int32_t* bt,
                        const int32_t* seqlens, const int32_t* indices, const sd_paged_desc& pd,
                        int B, int H, int k, float scale, uint16_t* out, float* lse,
                        const AttnPlan& p, float* part_o, float2* part_ml, int seqlen_cap,
                        cudaStream_t st) {
  using C = sd::AttnMmaCfg<DK, DV, MT>;
  const size_t smem = C::smem_bytes(vp != nullptr, p.slots_per_split);
  auto kern = sd::attn_split_mma_kernel<DK, DV, MT>;
  sd_status s = set_smem_limit(reinterpret_cast<const void*>(kern), smem);
  if (s != SD_OK) return s;
  const float scale_log2 = scale * 1.4426950408889634f;
  dim3 grid(p.n_splits, p.n_hb, B * pd.kv_heads);
  stage_mark(kStageAttn, 0, st);
  s = launch_k(kern, grid, dim3(C::THREADS), smem, st, reinterpret_cast<const __nv_bfloat16*>(q),
               reinterpret_cast<const __nv_bfloat16*>(kp), reinterpret_cast<const __nv_bfloat16*>(vp), bt, seqlens,
               indices, pd.num_pages, pd.page_size, pd.max_pages_per_req, pd.kv_heads, H, k, seqlen_cap, scale_log2,
               p.n_hb, p.n_splits, p.slots_per_split, part_o, part_ml);
  stage_mark(kStageAttn, 1, st);
  if (s != SD_OK) return s;
  stage_mark(kStageCombine, 0, st);
  s = launch_k(sd::attn_combine_kernel<DV>, dim3(B * H), dim3(128), 0, st, static_cast<const float*>(part_o),
               static_cast<const float2*>(part_ml), p.n_splits, reinterpret_cast<__nv_bfloat16*>(out), lse);
  stage_mark(kStageCombine, 1, st);
  return s;
}

// `rows_ready`: the top-k already resolved the selections to pool rows in the
// workspace's row array; otherwise a small kernel does it first. With
// n_layers > 1, q / out / lse hold n_layers x B requests (layer-major) that
// share the selection, seqlens and block table of the B real requests, and
// kp_layers[l] is layer l's latent cache; requests are "virtual" (layer * B +
// b) inside the kernels.
sd_status launch_attn_umma(const uint16_t* q, const uint16_t* const* kp_layers, int n_layers, const int32_t* bt,
                           const int32_t* seqlens, const int32_t* indices, const sd_paged_desc& pd, int B, int k,
                           float scale, uint16_t* out, float* lse, void* ws, int seqlen_cap, bool rows_ready,
                           cudaStream_t st) {
  using Lay = sd::AttnUmmaLayout;
  if (n_layers < 1 || n_layers > sd::kAuMaxLayers) return SD_ERR_UNSUPPORTED;
  const int Bv = n_layers * B;
  const size_t slots = static_cast<size_t>(sd::kAuRanges) + Bv;
  float* part_o = static_cast<float*>(ws);
  float2* part_ml = reinterpret_cast<float2*>(
      static_cast<char*>(ws) + align_up(slots * sd::kAuHeads * sd::kAuDv * sizeof(float)));
  int32_t* rows = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + sd::attn_umma_rows_offset(Bv));
  CUtensorMap tm_q;
  const uint64_t pool_rows = (uint64_t)pd.num_pages * pd.page_size;
  if (!encode_bf16_rows(&tm_q, q, sd::kAuDk, (uint64_t)Bv * sd::kAuHeads, sd::kAuDk * 2, 64, sd::kAuHalfHeads) ||
      pool_rows >= (1ull << 31))
    return SD_ERR_UNSUPPORTED;
  sd::AttnLayerKV kvl{};
  for (int l = 0; l < n_layers; ++l) {
    if (kp_layers[l] == nullptr || (reinterpret_cast<uintptr_t>(kp_layers[l]) & 15u) != 0) return SD_ERR_UNSUPPORTED;
    kvl.p[l] = reinterpret_cast<const __nv_bfloat16*>(kp_layers[l]);
  }
  sd_status s = set_smem_limit(reinterpret_cast<const void*>(sd::attn_mla_umma_kernel), Lay::kSmemAlloc);
  if (s != SD_OK) return s;
  const float scale_log2 = scale * 1.4426950408889634f;
  stage_mark(kStageAttn, 0, st);
  if (!rows_ready) {
    const dim3 grid((sd::attn_kpad(k) + 255) / 256, B);
    if ((s = launch_k(sd::attn_rows_kernel, grid, dim3(256), 0, st, indices, bt, seqlens, k, seqlen_cap, pd.page_size,
                      pd.max_pages_per_req, pd.num_pages, rows)) != SD_OK)
      return s;
  }
  s = launch_k(sd::attn_mla_umma_kernel, dim3(2 * sd::kAuRanges), dim3(sd::kAuThreads), Lay::kSmemAlloc, st, tm_q,
               kvl, seqlens, static_cast<const int32_t*>(rows), Bv, B, k, seqlen_cap, scale_log2, part_o, part_ml);
  stage_mark(kStageAttn, 1, st);
  if (s != SD_OK) return s;
  stage_mark(kStageCombine, 0, st);
  s = launch_k(sd::attn_mla_umma_combine_kernel, dim3(Bv * (sd::kAuHeads / sd::kAuCombineHeads)),
               dim3(32 * sd::kAuCombineHeads), 0, st, static_cast<const float*>(part_o),
               static_cast<const float2*>(part_ml), seqlens, Bv, B, k, seqlen_cap, sd::kAuRanges,
               reinterpret_cast<__nv_bfloat16*>(out), lse);
  stage_mark(kStageCombine, 1, st);
  return s;
}

sd_status launch_attn(const uint16_t* q, const uint16_t* kp, const uint16_t* vp, const int32_t* bt,
                      const int32_t* seqlens, const int32_t* indices, const sd_paged_desc& pd, int B,
                      int H, int Dk, int Dv, int k, float scale, uint16_t* out, float* lse,
                      void* ws, int seqlen_cap, cudaStream_t st, bool rows_ready = false) {
  if (B == 0) return SD_OK;
  if (umma_attn_fits(pd.kv_heads, H, Dk, Dv, vp != nullptr)) {
    const sd_status su =
        launch_attn_umma(q, &kp, 1, bt, seqlens, indices, pd, B, k, scale, out, lse, ws, seqlen_cap, rows_ready, st);
    if (su != SD_ERR_UNSUPPORTED) return su;  // else: pointers the TMA cannot map; take the mma.sync kernel
  }
  const AttnPlan p = attn_plan(B, pd.kv_heads, H, k);
  const size_t n = (size_t)B * H * p.n_splits;
  float* part_o = static_cast<float*>(ws);
  float2* part_ml = reinterpret_cast<float2*>(static_cast<char*>(ws) + align_up(sizeof(float) * n * Dv));
#define SD_ATTN(DK_, DV_)                                                                              \
  return p.mt == 2 ? launch_attn_t<DK_, DV_, 2>(q, kp, vp, bt, seqlens, indices, pd, B, H, k, scale, \
                                                out, lse, p, part_o, part_ml, seqlen_cap, st)         \
                   : launch_attn_t<DK_, DV_, 1>(q, kp, vp, bt, seqlens, indices, pd, B, H, k, scale, \
                                                out, lse, p, part_o, part_ml, seqlen_cap, st)
  if (Dk == 576) { SD_ATTN(576, 512); }
  if (Dk == 128) { SD_ATTN(128, 128); }
  SD_ATTN(64, 64);
#undef SD_ATTN
}

}  // namespace

extern "C" {

size_t sd_workspace_size(int32_t B, int32_t G, int32_t max_seqlen, int32_t k, int32_t H, int32_t Dv) {
  if (B < 0 || G <= 0 || max_seqlen < 0 || k <= 0 || H <= 0 || Dv <= 0 || H % G != 0) return 0;
  return scores_bytes(B, G, max_seqlen) + attn_bytes(B, G, H, k, Dv);
}

sd_status sd_indexer_topk_hinted(const int8_t* qi, const int32_t* w, const int8_t* ki_pages,
                                 const int32_t* block_table, const int32_t* seqlens, sd_paged_desc pd, int32_t B,
                                 int32_t Hi, int32_t Di, int32_t max_seqlen, int32_t k, const int32_t* hint,
                                 int32_t* indices, int32_t* scores, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  t_launches = 0;
  sd_status s = check_indexer_args(qi, w, ki_pages, block_table, seqlens, pd, B, Hi, Di, max_seqlen,
                                   k, indices);
  if (s != SD_OK) return s;
  if (hint != nullptr && hint == indices) return SD_ERR_INVALID_ARG;
  if (scores == nullptr) {
    if (!ws_ok(workspace, workspace_bytes, scores_bytes(B, pd.kv_heads, max_seqlen)))
      return SD_ERR_WORKSPACE;
    scores = static_cast<int32_t*>(workspace);
  }
  return launch_indexer_topk(qi, w, ki_pages, block_table, seqlens, pd, B, Hi, Di, max_seqlen, k,
                             indices, scores, static_cast<cudaStream_t>(stream), sd::RowMap{}, hint);
}

sd_status sd_indexer_topk(const int8_t* qi, const int32_t* w, const int8_t* ki_pages,
                          const int32_t* block_table, const int32_t* seqlens, sd_paged_desc pd,
                          int32_t B, int32_t Hi, int32_t Di, int32_t max_seqlen, int32_t k,
                          int32_t* indices, int32_t* scores, void* workspace, size_t workspace_bytes,
                          void* stream) {
  return sd_indexer_topk_hinted(qi, w, ki_pages, block_table, seqlens, pd, B, Hi, Di, max_seqlen, k, nullptr,
                                indices, scores, workspace, workspace_bytes, stream);
}

sd_status sd_sparse_attn(const uint16_t* q, const uint16_t* k_pages, const uint16_t* v_pages,
                         const int32_t* block_table, const int32_t* seqlens, const int32_t* indices,
                         sd_paged_desc pd, int32_t B, int32_t H, int32_t Dk, int32_t Dv, int32_t k,
                         float scale, uint16_t* out, float* lse, void* workspace,
                         size_t workspace_bytes, void* stream) {
  t_launches = 0;
  sd_status s = check_attn_args(q, k_pages, block_table, seqlens, indices, pd, B, H, Dk, Dv, k, scale,
                                out, v_pages != nullptr);
  if (s != SD_OK) return s;
  if (!ws_ok(workspace, workspace_bytes, attn_bytes(B, pd.kv_heads, H, k, Dv))) return SD_ERR_WORKSPACE;
  const int cap = pd.max_pages_per_req * pd.page_size;
  return launch_attn(q, k_pages, v_pages, block_table, seqlens, indices, pd, B, H, Dk, Dv, k, scale,
                     out, lse, workspace, cap, static_cast<cudaStream_t>(stream));
}

size_t sd_attn_layers_workspace_size(int32_t n_layers, int32_t B, int32_t G, int32_t k, int32_t H, int32_t Dv) {
  if (n_layers < 1 || B < 0 || G <= 0 || k <= 0 || H <= 0 || Dv <= 0) return 0;
  size_t bytes = attn_bytes(B, G, H, k, Dv);
  if (G == 1 && H == sd::kAuHeads && Dv == sd::kAuDv)
    bytes = std::max(bytes, align_up(sd::attn_umma_workspace(std::min(n_layers, (int32_t)sd::kAuMaxLayers) * B, k)));
  return bytes;
}

sd_status sd_sparse_attn_layers(const uint16_t* q, const uint16_t* const* k_pages, const uint16_t* const* v_pages,
                                int32_t n_layers, const int32_t* block_table, const int32_t* seqlens,
                                const int32_t* indices, sd_paged_desc pd, int32_t B, int32_t H, int32_t Dk,
                                int32_t Dv, int32_t k, float scale, uint16_t* out, float* lse, void* workspace,
                                size_t workspace_bytes, void* stream) {
  t_launches = 0;
  if (n_layers < 1 || k_pages == nullptr) return SD_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l)
    if (k_pages[l] == nullptr || (v_pages != nullptr && v_pages[l] == nullptr)) return SD_ERR_INVALID_ARG;
  sd_status s = check_attn_args(q, k_pages[0], block_table, seqlens, indices, pd, B, H, Dk, Dv, k, scale, out,
                                v_pages != nullptr);
  if (s != SD_OK) return s;
  if (!ws_ok(workspace, workspace_bytes, sd_attn_layers_workspace_size(n_layers, B, pd.kv_heads, k, H, Dv)))
    return SD_ERR_WORKSPACE;
  if (B == 0) return SD_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int cap = pd.max_pages_per_req * pd.page_size;
  const size_t q_layer = (size_t)B * H * Dk, o_layer = (size_t)B * H * Dv, l_layer = (size_t)B * H;
  int l0 = 0;
  if (v_pages == nullptr && umma_attn_fits(pd.kv_heads, H, Dk, Dv, false)) {
    // layers share the selection: one launch per group of up to kAuMaxLayers
    for (; l0 < n_layers; l0 += sd::kAuMaxLayers) {
      const int nl = std::min(n_layers - l0, (int)sd::kAuMaxLayers);
      s = launch_attn_umma(q + l0 * q_layer, k_pages + l0, nl, block_table, seqlens, indices, pd, B, k, scale,
                           out + l0 * o_layer, lse ? lse + l0 * l_layer : nullptr, workspace, cap, false, st);
      if (s == SD_ERR_UNSUPPORTED) break;  // pointers the TMA cannot map: one layer at a time below
      if (s != SD_OK) return s;
    }
  }
  const int launches = t_launches;
  for (int l = l0; l < n_layers; ++l) {
    s = launch_attn(q + l * q_layer, k_pages[l], v_pages ? v_pages[l] : nullptr, block_table, seqlens, indices, pd, B,
                    H, Dk, Dv, k, scale, out + l * o_layer, lse ? lse + l * l_layer : nullptr, workspace, cap, st);
    if (s != SD_OK) return s;
  }
  t_launches += launches;
  return SD_OK;
}

size_t sd_csr_workspace_size(int32_t B, int32_t G, int32_t max_selected, int32_t H, int32_t Dv) {
  if (B < 0 || G <= 0 || max_selected <= 0 || H <= 0 || Dv <= 0) return 0;
  return align_up((size_t)B * G * max_selected * sizeof(int32_t)) + attn_bytes(B, G, H, max_selected, Dv);
}

sd_status sd_sparse_attn_csr(const uint16_t* q, const uint16_t* k_pages, const uint16_t* v_pages,
                             const int32_t* block_table, const int32_t* seqlens, const int32_t* indices,
                             const int32_t* offsets, int32_t block_size, int32_t max_selected, sd_paged_desc pd,
                             int32_t B, int32_t H, int32_t Dk, int32_t Dv, float scale, uint16_t* out, float* lse,
                             void* workspace, size_t workspace_bytes, void* stream) {
  t_launches = 0;
  if (offsets == nullptr || block_size < 0) return SD_ERR_INVALID_ARG;
  // the packed entries may be empty: check the attention arguments with a placeholder for them
  sd_status s = check_attn_args(q, k_pages, block_table, seqlens, indices ? indices : offsets, pd, B, H, Dk, Dv,
                                max_selected, scale, out, v_pages != nullptr);
  if (s != SD_OK) return s;
  if (!ws_ok(workspace, workspace_bytes, sd_csr_workspace_size(B, pd.kv_heads, max_selected, H, Dv)))
    return SD_ERR_WORKSPACE;
  if (B == 0) return SD_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int cap = pd.max_pages_per_req * pd.page_size;
  int32_t* padded = static_cast<int32_t*>(workspace);
  void* attn_ws = static_cast<char*>(workspace) + align_up((size_t)B * pd.kv_heads * max_selected * sizeof(int32_t));
  s = launch_k(sd::csr_expand_kernel, dim3(B * pd.kv_heads), dim3(sd::kCsrThreads), 0, st,
               indices ? indices : offsets, offsets, block_size, seqlens, pd.kv_heads, max_selected, cap, padded);
  if (s != SD_OK) return s;
  const int launches = t_launches;
  s = launch_attn(q, k_pages, v_pages, block_table, seqlens, padded, pd, B, H, Dk, Dv, max_selected, scale, out, lse,
                  attn_ws, cap, st);
  t_launches += launches;
  return s;
}

}  // extern "C"

namespace {
struct TriPlan {
  int rows_per_req, e_max, moved, part, n_tiles, chunk, n_chunks;
  size_t off_tmax, off_keys, off_evict, off_sel, off_flags, flags_per_layer, total;
};
TriPlan tri_plan(int n_layers, int B, int G, int H, int D, int max_seqlen, int n_sink, int n_recent, int budget,
                 int mode, bool has_v) {
  TriPlan p{};
  p.rows_per_req = mode == SD_TRI_UNION ? 1 : G;
  p.e_max = std::max(0, max_seqlen - n_sink - n_recent);
  p.moved = budget + n_recent;
  p.part = (mode == SD_TRI_UNION ? G : 1) * D * 2;
  p.n_tiles = (p.e_max + sd::kTriTileTok - 1) / sd::kTriTileTok;
  p.chunk = std::max(1, std::min(sd::kTriMaxChunkTokens, sd::kTriChunkBytes / (p.part * (has_v ? 2 : 1))));
  p.n_chunks = (p.moved + p.chunk - 1) / p.chunk;
  const size_t rows = (size_t)B * p.rows_per_req;
  p.flags_per_layer = rows * p.n_chunks;
  p.off_tmax = align_up((size_t)B * H * p.e_max * sizeof(float));
  p.off_keys = p.off_tmax + align_up((size_t)B * H * p.n_tiles * sizeof(float));
  p.off_evict = p.off_keys + align_up(rows * p.e_max * sizeof(int32_t));
  p.off_sel = p.off_evict + align_up((size_t)B * sizeof(int32_t));
  p.off_flags = p.off_sel + align_up(rows * budget * sizeof(int32_t));
  p.total = p.off_flags + align_up((size_t)n_layers * p.flags_per_layer * sizeof(int32_t));
  return p;
}
bool tri_args_ok(int n_layers, int B, int G, int H, int D, int max_seqlen, int n_sink, int n_recent, int budget,
                 int mode) {
  return n_layers >= 1 && B >= 0 && G > 0 && H > 0 && H % G == 0 && max_seqlen >= 0 && n_sink >= 0 &&
         n_recent >= 0 && budget >= 1 &&
         (mode == SD_TRI_UNION || mode == SD_TRI_PER_HEAD || mode == SD_TRI_PER_LAYER_PER_HEAD);
}
// Co-resident CTAs of the compaction kernel on this device (its units wait on
// one another, so every CTA of its grid must be resident at once).
int tri_compact_grid() {
  static int grid = 0;
  if (grid == 0) {
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, sd::tri_compact_kernel, sd::kTriCompactThreads, 0) !=
            cudaSuccess)
      return 0;
    grid = sms * per_sm;
  }
  return grid;
}
template <int D, int QPK>
sd_status launch_tri_score(const uint16_t* q_cal, const uint16_t* kp, const int32_t* bt, const int32_t* seqlens,
                           const sd_paged_desc& pd, int B, int H, int cap, int n_sink, int n_recent, int e_max, float* z,
                           float* tmax, cudaStream_t st) {
  const dim3 grid((unsigned)((e_max + sd::kTriTileTok - 1) / sd::kTriTileTok), (unsigned)(B * pd.kv_heads));
  return launch_k(sd::tri_score_kernel<D, QPK>, grid, dim3(sd::kTriThreads), 0, st,
                  reinterpret_cast<const __nv_bfloat16*>(q_cal), reinterpret_cast<const __nv_bfloat16*>(kp), bt,
                  seqlens, H, pd.kv_heads, pd.page_size, pd.max_pages_per_req, pd.num_pages, cap, n_sink, n_recent,
                  e_max, z, tmax);
}

// One selection from the scores of layers [l0, l0 + nl) (folded by maximum),
// then every one of those layers compacted with it.
sd_status tri_select_compact(const uint16_t* const* q_cal, uint16_t* const* k_pages, uint16_t* const* v_pages, int l0,
                             int nl, const int32_t* block_table, const int32_t* seqlens, const sd_paged_desc& pd, int B,
                             int H, int D, int cap, int n_sink, int n_recent, int budget, int mode, const TriPlan& p,
                             int32_t* new_seqlens, char* ws, cudaStream_t st) {
  const int G = pd.kv_heads, qpk = H / G;
  float* z = reinterpret_cast<float*>(ws);
  float* tmax = reinterpret_cast<float*>(ws + p.off_tmax);
  int32_t* keys = reinterpret_cast<int32_t*>(ws + p.off_keys);
  int32_t* evict = reinterpret_cast<int32_t*>(ws + p.off_evict);
  int32_t* sel = reinterpret_cast<int32_t*>(ws + p.off_sel);
  int32_t* flags = reinterpret_cast<int32_t*>(ws + p.off_flags);
  const int rows = B * p.rows_per_req;
  sd_status s = SD_OK;
  if (p.e_max > 0) {
    for (int l = l0; l < l0 + nl; ++l) {
#define SD_TRI(D_, Q_)                                                                                            \
  s = launch_tri_score<D_, Q_>(q_cal[l], k_pages[l], block_table, seqlens, pd, B, H, cap, n_sink, n_recent, p.e_max, z, \
                               tmax, st)
      if (D == 64) {
        if (qpk == 1) SD_TRI(64, 1); else if (qpk == 2) SD_TRI(64, 2); else if (qpk == 4) SD_TRI(64, 4); else SD_TRI(64, 8);
      } else {
        if (qpk == 1) SD_TRI(128, 1); else if (qpk == 2) SD_TRI(128, 2); else if (qpk == 4) SD_TRI(128, 4); else SD_TRI(128, 8);
      }
#undef SD_TRI
      if (s != SD_OK) return s;
      const dim3 rgrid((unsigned)((p.e_max + sd::kTriReduceThreads - 1) / sd::kTriReduceThreads), (unsigned)rows);
      if ((s = launch_k(sd::tri_reduce_kernel, rgrid, dim3(sd::kTriReduceThreads), 0, st, static_cast<const float*>(z),
                        static_cast<const float*>(tmax), seqlens, H, G, p.rows_per_req, cap, n_sink, n_recent,
                        p.e_max, keys, evict, flags + (size_t)l * p.flags_per_layer, p.n_chunks, l > l0 ? 1 : 0)) !=
          SD_OK)
        return s;
    }
    if ((s = launch_topk(keys, evict, sel, B, p.rows_per_req, p.e_max, p.e_max, budget, sd::RowMap{}, nullptr, st)) !=
        SD_OK)
      return s;
  }
  const int grid = tri_compact_grid();
  if (grid <= 0) return cuda_check(cudaGetLastError());
  const long long units = (long long)rows * p.n_chunks;
  for (int l = l0; l < l0 + nl; ++l) {
    if ((s = launch_k(sd::tri_compact_kernel, dim3((unsigned)std::max(1LL, std::min<long long>(grid, units))),
                      dim3(sd::kTriCompactThreads), 0, st, reinterpret_cast<uint8_t*>(k_pages[l]),
                      reinterpret_cast<uint8_t*>(v_pages ? v_pages[l] : nullptr), block_table, seqlens,
                      static_cast<const int32_t*>(sel), p.rows_per_req, pd.page_size, pd.max_pages_per_req,
                      pd.num_pages, cap, n_sink, n_recent, budget, p.part, G * D * 2, p.chunk, p.n_chunks, rows,
                      flags + (size_t)l * p.flags_per_layer, new_seqlens,
                      g_tri_wait_limit.load(std::memory_order_relaxed))) != SD_OK)
      return s;
  }
  return SD_OK;
}
}  // namespace

extern "C" {

size_t sd_tri_layers_workspace_size(int32_t n_layers, int32_t B, int32_t G, int32_t H, int32_t D, int32_t max_seqlen,
                                    int32_t n_sink, int32_t n_recent, int32_t budget, int32_t mode, int32_t has_v) {
  if (!tri_args_ok(n_layers, B, G, H, D, max_seqlen, n_sink, n_recent, budget, mode)) return 0;
  return tri_plan(n_layers, B, G, H, D, max_seqlen, n_sink, n_recent, budget, mode, has_v != 0).total;
}

size_t sd_tri_workspace_size(int32_t B, int32_t G, int32_t H, int32_t D, int32_t max_seqlen, int32_t n_sink,
                             int32_t n_recent, int32_t budget, int32_t mode, int32_t has_v) {
  return sd_tri_layers_workspace_size(1, B, G, H, D, max_seqlen, n_sink, n_recent, budget, mode, has_v);
}

sd_status sd_tri_compact_layers(const uint16_t* const* q_cal, uint16_t* const* k_pages, uint16_t* const* v_pages,
                                int32_t n_layers, const int32_t* block_table, const int32_t* seqlens, sd_paged_desc pd,
                                int32_t B, int32_t H, int32_t D, int32_t max_seqlen, int32_t n_sink, int32_t n_recent,
                                int32_t budget, int32_t mode, int32_t* new_seqlens, void* workspace,
                                size_t workspace_bytes, void* stream) {
  t_launches = 0;
  if (n_layers < 1 || !q_cal || !k_pages || !geom_ok(pd) || (B > 0 && (!block_table || !seqlens || !new_seqlens)))
    return SD_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l) {
    if (!q_cal[l] || !k_pages[l] || (v_pages && !v_pages[l])) return SD_ERR_INVALID_ARG;
    // pool rows are copied in 16-byte units
    if ((reinterpret_cast<uintptr_t>(k_pages[l]) & 15u) != 0 ||
        (v_pages && (reinterpret_cast<uintptr_t>(v_pages[l]) & 15u) != 0))
      return SD_ERR_INVALID_ARG;
  }
  const int G = pd.kv_heads;
  if (!tri_args_ok(n_layers, B, G, H, D, max_seqlen, n_sink, n_recent, budget, mode)) return SD_ERR_INVALID_ARG;
  const int qpk = H / G;
  if ((D != 64 && D != 128) || (qpk != 1 && qpk != 2 && qpk != 4 && qpk != 8) || budget > kMaxK)
    return SD_ERR_UNSUPPORTED;
  // grid y of the score and reduce passes; heads of the reduce
  if ((long long)B * G > 65535 || H > sd::kTriMaxHeads) return SD_ERR_UNSUPPORTED;
  const bool has_v = v_pages != nullptr;
  if ((mode == SD_TRI_UNION ? G : 1) * D * 2 * (has_v ? 2 : 1) > sd::kTriChunkBytes) return SD_ERR_UNSUPPORTED;
  const TriPlan p = tri_plan(n_layers, B, G, H, D, max_seqlen, n_sink, n_recent, budget, mode, has_v);
  if (!ws_ok(workspace, workspace_bytes, p.total)) return SD_ERR_WORKSPACE;
  if (B == 0) return SD_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  const int cap = std::min(max_seqlen, pd.max_pages_per_req * pd.page_size);
  if (mode == SD_TRI_PER_LAYER_PER_HEAD) {  // an independent per-head selection in every layer
    for (int l = 0; l < n_layers; ++l) {
      const sd_status s = tri_select_compact(q_cal, k_pages, v_pages, l, 1, block_table, seqlens, pd, B, H, D, cap,
                                             n_sink, n_recent, budget, mode, p, new_seqlens, ws, st);
      if (s != SD_OK) return s;
    }
    return SD_OK;
  }
  return tri_select_compact(q_cal, k_pages, v_pages, 0, n_layers, block_table, seqlens, pd, B, H, D, cap, n_sink,
                            n_recent, budget, mode, p, new_seqlens, ws, st);
}

sd_status sd_tri_compact(const uint16_t* q_cal, uint16_t* k_pages, uint16_t* v_pages, const int32_t* block_table,
                         const int32_t* seqlens, sd_paged_desc pd, int32_t B, int32_t H, int32_t D, int32_t max_seqlen,
                         int32_t n_sink, int32_t n_recent, int32_t budget, int32_t mode, int32_t* new_seqlens,
                         void* workspace, size_t workspace_bytes, void* stream) {
  const uint16_t* q1[1] = {q_cal};
  uint16_t* k1[1] = {k_pages};
  uint16_t* v1[1] = {v_pages};
  return sd_tri_compact_layers(q1, k1, v_pages ? v1 : nullptr, 1, block_table, seqlens, pd, B, H, D, max_seqlen,
                               n_sink, n_recent, budget, mode, new_seqlens, workspace, workspace_bytes, stream);
}

sd_status sd_decode_step_hinted(const int8_t* qi, const int32_t* w, const int8_t* ki_pages, const uint16_t* q,
                         const uint16_t* k_pages, const uint16_t* v_pages, const int32_t* block_table,
                         const int32_t* seqlens, sd_paged_desc pd, int32_t B, int32_t Hi, int32_t Di,
                         int32_t H, int32_t Dk, int32_t Dv, int32_t max_seqlen, int32_t k, float scale, const int32_t* hint,
                         int32_t* indices, int32_t* scores, uint16_t* out, float* lse, void* workspace,
                         size_t workspace_bytes, void* stream) {
  t_launches = 0;
  sd_status s = check_indexer_args(qi, w, ki_pages, block_table, seqlens, pd, B, Hi, Di, max_seqlen,
                                   k, indices);
  if (s != SD_OK) return s;
  s = check_attn_args(q, k_pages, block_table, seqlens, indices, pd, B, H, Dk, Dv, k, scale, out,
                      v_pages != nullptr);
  if (s != SD_OK) return s;
  if (hint != nullptr && hint == indices) return SD_ERR_INVALID_ARG;
  const size_t sb = scores_bytes(B, pd.kv_heads, max_seqlen);
  if (!ws_ok(workspace, workspace_bytes, sd_workspace_size(B, pd.kv_heads, max_seqlen, k, H, Dv)))
    return SD_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* sc = scores ? scores : static_cast<int32_t*>(workspace);
  void* attn_ws = static_cast<char*>(workspace) + sb;
  // With the tensor-core attention, the top-k also resolves each selection to
  // its pool row (one block-table load per selected token, off the
  // attention's gather path).
  const bool umma = umma_attn_fits(pd.kv_heads, H, Dk, Dv, v_pages != nullptr) && B > 0 &&
                    (reinterpret_cast<uintptr_t>(q) & 15u) == 0 && (reinterpret_cast<uintptr_t>(k_pages) & 15u) == 0;
  sd::RowMap rm{};
  if (umma)
    rm = sd::RowMap{reinterpret_cast<int32_t*>(static_cast<char*>(attn_ws) + sd::attn_umma_rows_offset(B)),
                    block_table, pd.page_size, pd.max_pages_per_req, pd.num_pages, sd::attn_kpad(k)};
  s = launch_indexer_topk(qi, w, ki_pages, block_table, seqlens, pd, B, Hi, Di, max_seqlen, k, indices,
                          sc, st, rm, hint);
  if (s != SD_OK) return s;
  const int launches = t_launches;
  const int cap = std::min(max_seqlen, pd.max_pages_per_req * pd.page_size);
  s = launch_attn(q, k_pages, v_pages, block_table, seqlens, indices, pd, B, H, Dk, Dv, k, scale, out,
                  lse, attn_ws, cap, st, umma);
  t_launches += launches;
  return s;
}

sd_status sd_decode_step(const int8_t* qi, const int32_t* w, const int8_t* ki_pages, const uint16_t* q,
                         const uint16_t* k_pages, const uint16_t* v_pages, const int32_t* block_table,
                         const int32_t* seqlens, sd_paged_desc pd, int32_t B, int32_t Hi, int32_t Di,
                         int32_t H, int32_t Dk, int32_t Dv, int32_t max_seqlen, int32_t k, float scale,
                         int32_t* indices, int32_t* scores, uint16_t* out, float* lse, void* workspace,
                         size_t workspace_bytes, void* stream) {
  return sd_decode_step_hinted(qi, w, ki_pages, q, k_pages, v_pages, block_table, seqlens, pd, B, Hi, Di, H, Dk, Dv,
                               max_seqlen, k, scale, nullptr, indices, scores, out, lse, workspace, workspace_bytes,
                               stream);
}

sd_status sd_set_stage_events(void* const* events, int32_t n) {
  if (n < 0 || n > 4 || (n > 0 && events == nullptr)) return SD_ERR_INVALID_ARG;
  for (int i = 0; i < 2 * n; ++i) {
    if (events[i] == nullptr) return SD_ERR_INVALID_ARG;
    t_stage_events[i] = static_cast<cudaEvent_t>(events[i]);
  }
  t_stage_count = n;
  return SD_OK;
}

sd_status sd_set_wait_limit(int32_t polls) {
  if (polls > static_cast<int32_t>(sd::kTriWaitLimit)) return SD_ERR_INVALID_ARG;
  g_tri_wait_limit.store(polls < 0 ? sd::kTriWaitLimit : static_cast<uint32_t>(polls), std::memory_order_relaxed);
  return SD_OK;
}

sd_status sd_get_device_errors(uint32_t* bits, int32_t clear) {
  if (!bits) return SD_ERR_INVALID_ARG;
  sd_status s = cuda_check(cudaDeviceSynchronize());
  if (s != SD_OK) return s;
  s = cuda_check(cudaMemcpyFromSymbol(bits, sd::g_error_bits, sizeof(uint32_t)));
  if (s != SD_OK || !clear) return s;
  const uint32_t zero = 0;
  return cuda_check(cudaMemcpyToSymbol(sd::g_error_bits, &zero, sizeof(uint32_t)));
}

const char* sd_status_str(sd_status status) {
  switch (status) {
    case SD_OK: return "SD_OK";
    case SD_ERR_INVALID_ARG: return "SD_ERR_INVALID_ARG";
    case SD_ERR_UNSUPPORTED: return "SD_ERR_UNSUPPORTED";
    case SD_ERR_WORKSPACE: return "SD_ERR_WORKSPACE";
    case SD_ERR_CUDA: return "SD_ERR_CUDA";
  }
  return "SD_ERR_UNKNOWN";
}

#ifdef SD_PROBE
// Probe builds only: copies the probe slots (u64 ns, [4][1024][16][64], 0 =
// not recorded) to host memory if dst is not NULL, then clears them.
int64_t sd_probe_read(void* dst, int64_t max_bytes) {
  const size_t n = sizeof(sd::g_probe);
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  if (dst != nullptr && max_bytes >= (int64_t)n && cudaMemcpyFromSymbol(dst, sd::g_probe, n) != cudaSuccess) return -1;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, sd::g_probe) != cudaSuccess || cudaMemset(p, 0, n) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess)
    return -1;
  return (int64_t)n;
}
#endif

int32_t sd_last_cuda_error(void) { return t_last_cuda_error; }
int32_t sd_last_launch_count(void) { return t_launches; }
int32_t sd_version(void) { return (0 << 16) | 7; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free indexer + top-k. The scores go to a fixed scratch array in
// this library's device image instead of a caller workspace. The host-side name
// g_noalloc_scores is a stand-in, not a device address. Host code must never
// hand it to a kernel. Each device's real address is looked up once, with
// that device current, and cached here.
// ---------------------------------------------------------------------------
static __device__ __align__(256) int32_t g_noalloc_scores[SD_NOALLOC_MAX_SCORES];

namespace {
constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mutex;
int32_t* g_noalloc_addr[kNoallocMaxDevices] = {};

// The current device's address of g_noalloc_scores. Outside stream capture it
// is looked up again on every call (a device reset reloads the module at
// another address, so a remembered one could be stale); under capture the
// remembered address is used, since a lookup could load the module.
sd_status noalloc_scores_for_current_device(cudaStream_t st, int32_t** out) {
  int dev = 0;
  sd_status s = cuda_check(cudaGetDevice(&dev));
  if (s != SD_OK) return s;
  if (dev < 0 || dev >= kNoallocMaxDevices) return SD_ERR_UNSUPPORTED;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  s = cuda_check(cudaStreamIsCapturing(st, &cap));
  if (s != SD_OK) return s;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    s = cuda_check(cudaGetSymbolAddress(&p, g_noalloc_scores));
    if (s != SD_OK) return s;
    g_noalloc_addr[dev] = static_cast<int32_t*>(p);
  } else if (g_noalloc_addr[dev] == nullptr) {
    return SD_ERR_INVALID_ARG;  // first call on this device under capture
  }
  *out = g_noalloc_addr[dev];
  return SD_OK;
}
}  // namespace

extern "C" sd_status sd_indexer_topk_noalloc(const int8_t* qi, const int32_t* w, const int8_t* ki_pages,
                                             const int32_t* block_table, const int32_t* seqlens,
                                             sd_paged_desc pd, int32_t B, int32_t Hi, int32_t Di,
                                             int32_t max_seqlen, int32_t k, int32_t* indices,
                                             void* stream) {
  t_launches = 0;
  sd_status s = check_indexer_args(qi, w, ki_pages, block_table, seqlens, pd, B, Hi, Di, max_seqlen,
                                   k, indices);
  if (s != SD_OK) return s;
  if ((size_t)B * pd.kv_heads * (size_t)max_seqlen > (size_t)SD_NOALLOC_MAX_SCORES) return SD_ERR_WORKSPACE;
  int32_t* scores = nullptr;
  s = noalloc_scores_for_current_device(static_cast<cudaStream_t>(stream), &scores);
  if (s != SD_OK) return s;
  // Scores are written for every t < seqlens[b] before top-k reads them, so
  // nothing left over from an earlier call is ever read.
  return launch_indexer_topk(qi, w, ki_pages, block_table, seqlens, pd, B, Hi, Di, max_seqlen, k,
                             indices, scores, static_cast<cudaStream_t>(stream));
}
