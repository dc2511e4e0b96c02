// Alternative index layouts for the selected tokens, the algorithm-independent
// indexing data of the unified sparse runtime ("Unify sparse attention
// framework with clean backend interfaces", review of the runtime parameters:
// sparse_attn_offsets and sparse_attn_indices_block_size).
//
// CSR: the selections of all (request, KV head) rows r = b * G + g are packed
// in one flat array; offsets[r] .. offsets[r + 1] delimit row r's entries.
// Block-sized indices: an entry e selects the block_size consecutive tokens
// e * bs .. e * bs + bs - 1 (bs = max(block_size, 1)).
//
// csr_expand_kernel turns a CSR row into the padded per-row form every
// attention path reads: the valid tokens of the expansion, in list order,
// first, then -1. A token is valid when its entry is >= 0 and it is below the
// request's seqlen (tokens of a block past the seqlen are dropped; an entry
// whose whole block lies past it flags SD_DEVERR_INDEX). Only the first
// min(kmax, L_b) valid tokens are kept, which is what the attention reads;
// more than that flags SD_DEVERR_INDEX. Duplicates are kept as listed.
#pragma once

#include "sd_common.cuh"

namespace sd {

constexpr int kCsrThreads = 256;
constexpr int kCsrPerThread = 8;  // consecutive expanded slots per thread and chunk

__global__ void __launch_bounds__(kCsrThreads) csr_expand_kernel(const int32_t* __restrict__ indices,
                                                                 const int32_t* __restrict__ offsets, int block_size,
                                                                 const int32_t* __restrict__ seqlens, int G, int kmax,
                                                                 int seqlen_cap, int32_t* __restrict__ out) {
  pdl_wait();  // inputs come from earlier work in the stream
  pdl_trigger();
  __shared__ int warp_tot[kCsrThreads / 32];
  const int r = blockIdx.x;
  const int b = r / G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bs = max(block_size, 1);
  const int L = checked_seqlen(seqlens, b, seqlen_cap);
  const int o0 = offsets[r], o1 = offsets[r + 1];
  if (o1 < o0 && tid == 0) raise_error(SD_DEVERR_INDEX);
  const long long n = o1 > o0 ? (long long)(o1 - o0) * bs : 0;  // expanded slots
  const int cap = min(kmax, L);
  int32_t* dst = out + (size_t)r * kmax;
  long long written = 0;  // valid tokens found so far (uniform)
  constexpr int kChunk = kCsrThreads * kCsrPerThread;
  for (long long base = 0; base < n && written <= cap; base += kChunk) {
    int tok[kCsrPerThread];
    int cnt = 0;
#pragma unroll
    for (int i = 0; i < kCsrPerThread; ++i) {
      const long long s = base + tid * kCsrPerThread + i;
      tok[i] = -1;
      if (s < n) {
        const int e = indices[o0 + static_cast<int>(s / bs)];
        const int u = static_cast<int>(s % bs);
        if (e >= 0) {
          const long long t = (long long)e * bs + u;
          if ((long long)e * bs >= L) {
            if (u == 0) raise_error(SD_DEVERR_INDEX);
          } else if (t < L) {
            tok[i] = static_cast<int>(t);
          }
        }
      }
      cnt += tok[i] >= 0;
    }
    // block-wide exclusive scan of the per-thread counts (list order is kept)
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < kCsrThreads / 32; ++w) {
      before += w < warp ? warp_tot[w] : 0;
      total += warp_tot[w];
    }
    long long pos = written + before + incl - cnt;
#pragma unroll
    for (int i = 0; i < kCsrPerThread; ++i) {
      if (tok[i] >= 0) {
        if (pos < cap) dst[pos] = tok[i];
        ++pos;
      }
    }
    written += total;
    __syncthreads();  // warp_tot is rewritten by the next chunk
  }
  if (written > cap && tid == 0) raise_error(SD_DEVERR_INDEX);
  for (long long s = min(written, (long long)cap) + tid; s < kmax; s += kCsrThreads) dst[s] = -1;
}

}  // namespace sd
