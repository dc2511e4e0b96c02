// Per-row top-k of int32 indexer scores by radix select, then an ordered
// compaction that writes the chosen tokens in ascending order.
//
// Order: score descending, ties to the lower token index (the deterministic
// tie settlement the TriAttention selector tests for, "Add TriAttention
// KV-cache compression method", Test Plan). The output row is the persistent
// top-k buffer the attention consumes ("Overlap DSA heuristic prev_topk
// write-back...", Description): min(k, L) ascending token ids, then -1.
//
// Radix select on the order-preserving key u = s ^ 0x80000000 (signed ->
// unsigned): four 8-bit passes from the top digit narrow the candidate prefix
// until the k-th largest key T is known, together with how many keys equal to
// T must be taken (need_eq). The compaction pass then walks the row in token
// order: a token is taken if u > T, or u == T and fewer than need_eq equal keys
// precede it. Block-wide ballot scans give each taken token its output slot.
#pragma once

#include "sd_common.cuh"

namespace sd {

constexpr int kTopkThreads = 1024;
constexpr int kTopkWarps = kTopkThreads / 32;

__device__ __forceinline__ uint32_t score_key(int32_t s) { return static_cast<uint32_t>(s) ^ 0x80000000u; }

// Exclusive block scan of a 0/1 flag; returns this thread's prefix and, through
// `total`, the block total. `warp_sums` holds kTopkWarps words of scratch.
__device__ __forceinline__ int block_excl_scan_flag(bool flag, uint32_t* warp_sums, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t m = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(m & ((1u << lane) - 1u));
  if (lane == 0) warp_sums[warp] = __popc(m);
  __syncthreads();
  if (warp == 0) {
    const uint32_t v = warp_sums[lane];
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    warp_sums[lane] = incl - v;                      // exclusive
    if (lane == 31) warp_sums[kTopkWarps] = incl;    // total
  }
  __syncthreads();
  const int r = static_cast<int>(warp_sums[warp]) + in_warp;
  total = static_cast<int>(warp_sums[kTopkWarps]);
  __syncthreads();                                   // scratch reused by the next scan
  return r;
}

__global__ void __launch_bounds__(kTopkThreads) topk_radix_kernel(
    const int32_t* __restrict__ scores, const int32_t* __restrict__ seqlens, int32_t* __restrict__ indices,
    int G, int max_seqlen, int seqlen_cap, int k, RowMap rm) {
  pdl_wait();  // inputs come from earlier work in the stream
  pdl_trigger();

  __shared__ uint32_t hist[256];
  __shared__ uint32_t scan_scratch[kTopkWarps + 1];
  __shared__ int sel_digit, sel_remaining;

  const int row = blockIdx.x;  // b * G + g
  const int b = row / G;
  const int L = checked_seqlen(seqlens, b, seqlen_cap);
  const int32_t* s = scores + (size_t)row * max_seqlen;
  int32_t* out = indices + (size_t)row * k;
  int2 pc = make_int2(-1, 0);  // last block-table lookup (row ids)

  if (L <= k) {  // everything is selected: 0..L-1 then -1
    const int n = rm.rows != nullptr ? max(k, rm.kpad) : k;
    for (int i = threadIdx.x; i < n; i += kTopkThreads) {
      if (i < k) out[i] = i < L ? i : -1;
      rm.put(row, b, i, i < L ? i : -1, pc);
    }
    return;
  }


  uint32_t prefix = 0, prefix_mask = 0;
  int remaining = k;  // how many still to take among keys that match `prefix`
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = threadIdx.x; i < 256; i += kTopkThreads) hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < L; i += kTopkThreads) {
      const uint32_t u = score_key(s[i]);
      if ((u & prefix_mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l owns digits 255-8l .. 248-8l (descending); find the digit where
      // the count of larger-or-equal digits first reaches `remaining`.
      const int lane = threadIdx.x;
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[255 - 8 * lane - j];
        sum += c[j];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      uint32_t acc = incl - sum;  // keys with a larger digit than this lane's range
      const uint32_t need = static_cast<uint32_t>(remaining);
      if (acc < need && acc + sum >= need) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (acc < need && acc + c[j] >= need) {
            sel_digit = 255 - 8 * lane - j;
            sel_remaining = static_cast<int>(need - acc);
          }
          acc += c[j];
        }
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(sel_digit) << shift;
    prefix_mask |= 255u << shift;
    remaining = sel_remaining;
    __syncthreads();
  }
  const uint32_t T = prefix;
  const int need_eq = remaining;

  int taken_eq = 0, written = 0;
  for (int base = 0; base < L; base += kTopkThreads) {
    const int i = base + threadIdx.x;
    const bool valid = i < L;
    const uint32_t u = valid ? score_key(s[i]) : 0u;
    const bool gt = valid && u > T;
    const bool eq = valid && u == T;
    int eq_total;
    const int eq_rank = block_excl_scan_flag(eq, scan_scratch, eq_total) + taken_eq;
    const bool take = gt || (eq && eq_rank < need_eq);
    int take_total;
    const int pos = block_excl_scan_flag(take, scan_scratch, take_total) + written;
    if (take) out[pos] = i;
    taken_eq += eq_total;
    written += take_total;
  }
  if (rm.rows != nullptr) {
    __syncthreads();  // the output above is complete
    for (int i = threadIdx.x; i < rm.kpad; i += kTopkThreads) rm.put(row, b, i, i < k ? out[i] : -1, pc);
  }
}

}  // namespace sd
