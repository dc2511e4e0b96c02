// Indexer scores on CUDA cores (dp4a), any supported (G, Hi, Di).
//
//   s[b,g,t] = sum_h w[b,g,h] * max(0, sum_d qi[b,g,h,d] * ki[t,g,d])
//
// Keys are read in place from the paged int8 pool through the block table
// (the pages' "direct paged-pool scoring ... no Torch gather" of the TriAttention
// scorer, Key Design Decisions). This kernel is the general path: it serves
// thin indexers (few heads per KV head, as in per-head selection) where the
// [Hi x Di] x [Di x L] contraction is too narrow for tensor cores and the
// stream of keys is the bound. Wide indexers (Hi = 64, Di = 128) go to the
// tcgen05 kernel instead.
//
// One thread scores one (token, KV head) pair; consecutive threads read
// consecutive (slot, g) rows, so each warp reads a contiguous span of the page.
#pragma once

#include "sd_common.cuh"

namespace sd {

constexpr int kIdxThreads = 256;
constexpr int kIdxTokensPerCta = 256;

template <int DI>
__global__ void __launch_bounds__(kIdxThreads) indexer_dp4a_kernel(
    const int8_t* __restrict__ qi, const int32_t* __restrict__ w, const int8_t* __restrict__ ki_pages,
    const int32_t* __restrict__ block_table, const int32_t* __restrict__ seqlens,
    int32_t* __restrict__ scores, int num_pages, int page_size, int max_pages, int G, int Hi,
    int max_seqlen) {
  pdl_wait();  // inputs come from earlier work in the stream
  pdl_trigger();

  constexpr int W4 = DI / 4;      // int32 words per key row
  extern __shared__ int32_t smem_i32[];
  const int b = blockIdx.y;
  const int t0 = blockIdx.x * kIdxTokensPerCta;
  const int cap = min(max_seqlen, max_pages * page_size);
  const int L = checked_seqlen(seqlens, b, cap);
  if (t0 >= L) return;

  // q rows for all KV heads of this request, per-g stride padded by one word
  // so that threads of different g hit different banks.
  const int gstride = Hi * W4 + 1;
  int32_t* sq = smem_i32;
  int32_t* sw = smem_i32 + G * gstride;
  const int32_t* qw = reinterpret_cast<const int32_t*>(qi + (size_t)b * G * Hi * DI);
  for (int i = threadIdx.x; i < G * Hi * W4; i += kIdxThreads) {
    const int g = i / (Hi * W4), r = i % (Hi * W4);
    sq[g * gstride + r] = qw[i];
  }
  for (int i = threadIdx.x; i < G * Hi; i += kIdxThreads) sw[i] = w[(size_t)b * G * Hi + i];
  __syncthreads();

  const int t_end = min(L, t0 + kIdxTokensPerCta);
  const int npairs = (t_end - t0) * G;
  for (int p = threadIdx.x; p < npairs; p += kIdxThreads) {
    const int t = t0 + p / G;
    const int g = p % G;
    const int page = block_table[(size_t)b * max_pages + t / page_size];
    int32_t* dst = scores + ((size_t)b * G + g) * max_seqlen + t;
    if (page < 0 || page >= num_pages) {
      raise_error(SD_DEVERR_PAGE);
      *dst = INT32_MIN;
      continue;
    }
    const int8_t* row = ki_pages + (((size_t)page * page_size + (t % page_size)) * G + g) * DI;
    int32_t kv[W4];
#pragma unroll
    for (int j = 0; j < W4 / 4; ++j) {
      const int4 v = __ldg(reinterpret_cast<const int4*>(row) + j);
      kv[4 * j + 0] = v.x;
      kv[4 * j + 1] = v.y;
      kv[4 * j + 2] = v.z;
      kv[4 * j + 3] = v.w;
    }
    const int32_t* qg = sq + g * gstride;
    int32_t acc = 0;
    for (int h = 0; h < Hi; ++h) {
      int32_t dot = 0;
#pragma unroll
      for (int j = 0; j < W4; ++j) dot = __dp4a(qg[h * W4 + j], kv[j], dot);
      acc += sw[g * Hi + h] * max(dot, 0);
    }
    *dst = acc;
  }
}

inline size_t indexer_dp4a_smem(int G, int Hi, int Di) {
  return sizeof(int32_t) * ((size_t)G * (Hi * (Di / 4) + 1) + (size_t)G * Hi);
}

}  // namespace sd
