// Per-row top-k of int32 indexer scores with one thread-block cluster per row.
//
// Same result as topk_radix_kernel (score descending, ties to the lower token,
// output in ascending token order, -1 padded), organised for B200:
//   - a row of L scores is split over a cluster of CS CTAs (CS <= 8); each CTA
//     copies its slice (512 threads x 16 or 32 scores) once from L2 into shared
//     memory and never touches global memory again until it writes its part of
//     the output;
//   - a cluster-wide min/max fixes the highest bit in which the keys differ,
//     so radix passes start there (for scores of one row that is ~22 bits:
//     two 11-bit passes, not four 8-bit ones);
//   - each pass builds a 2048-bin histogram per CTA in shared memory; the CTAs
//     read each other's histograms through distributed shared memory, so every
//     CTA knows the threshold digit without a global round trip;
//   - the final pass is an ordered compaction: per-thread counts of "greater"
//     and "equal to the threshold" keys, one block scan, one cluster exchange
//     of CTA totals, and each thread writes its picks in token order.
// No CTA waits on another except at hardware cluster barriers.
#pragma once

#include <cooperative_groups.h>

#include "sd_common.cuh"

namespace sd {

namespace cg = cooperative_groups;

constexpr int kTkThreads = 512;
constexpr int kTkBinsBits = 11;
constexpr int kTkBins = 1 << kTkBinsBits;
constexpr int kTkMaxCluster = 8;

// PER: scores per thread (16 or 32); a CTA holds a slice of 512 * PER scores.
template <int PER>
struct TopkClusterSmem {
  static constexpr int kStride = PER + 1;       // padded per-thread chunk (words)
  uint32_t keys[kTkThreads * kStride];          // thread t's chunk at t*(PER+1) (bank-conflict free)
  uint32_t hist[kTkBins];                       // this CTA's histogram (read by the cluster)
  uint32_t total[kTkBins];                      // cluster-wide histogram
  uint32_t red[kTkThreads / 32 * 2 + 8];        // block reduction / scan scratch
  uint32_t cta_vals[4];                         // values this CTA publishes to the cluster
  uint32_t found[2];                            // threshold digit, remaining
  uint32_t mark[kTkThreads * PER / 32];         // hint tokens of this CTA's slice (one bit each)
  uint32_t hvals[4];                            // hint bounds this CTA publishes
};

// Block-wide exclusive scan of 32-bit values (512 threads); returns the prefix,
// writes the total to *total.
__device__ __forceinline__ uint32_t tk_block_excl_scan(uint32_t v, uint32_t* scratch, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = lane < kTkThreads / 32 ? scratch[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    if (lane < kTkThreads / 32) scratch[lane] = wi - w;
    if (lane == 31) scratch[kTkThreads / 32] = wi;
  }
  __syncthreads();
  const uint32_t r = scratch[warp] + incl - v;
  *total = scratch[kTkThreads / 32];
  __syncthreads();
  return r;
}

__device__ __forceinline__ uint32_t tk_block_reduce(uint32_t v, uint32_t* scratch, bool is_max) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint32_t n = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? max(v, n) : min(v, n);
  }
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < kTkThreads / 32 ? scratch[lane] : (is_max ? 0u : 0xffffffffu);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint32_t n = __shfl_xor_sync(0xffffffffu, v, o);
      v = is_max ? max(v, n) : min(v, n);
    }
    if (lane == 0) scratch[kTkThreads / 32] = v;
  }
  __syncthreads();
  v = scratch[kTkThreads / 32];
  __syncthreads();
  return v;
}

template <int PER>
__global__ void __launch_bounds__(kTkThreads, 2) topk_cluster_kernel(
    const int32_t* __restrict__ scores, const int32_t* __restrict__ seqlens, int32_t* __restrict__ indices,
    int G, int max_seqlen, int seqlen_cap, int k, RowMap rm, const int32_t* __restrict__ hint) {
  pdl_wait();  // inputs come from earlier work in the stream
  pdl_trigger();

  constexpr int kTkPerThread = PER;
  constexpr int kTkChunkStride = PER + 1;
  extern __shared__ __align__(16) uint8_t tk_smem_raw[];
  TopkClusterSmem<PER>& sm = *reinterpret_cast<TopkClusterSmem<PER>*>(tk_smem_raw);
  cg::cluster_group cluster = cg::this_cluster();
  const int CS = static_cast<int>(cluster.num_blocks());
  const int crank = static_cast<int>(cluster.block_rank());
  const int row = blockIdx.y;
  const int b = row / G;
  const int tid = threadIdx.x;
  const int L = checked_seqlen(seqlens, b, seqlen_cap);
  int32_t* out = indices + (size_t)row * k;
  int2 pc = make_int2(-1, 0);  // last block-table lookup (row ids)

  if (L <= k) {  // uniform over the cluster: no cluster barrier is reached
    const int n = rm.rows != nullptr ? max(k, rm.kpad) : k;
    for (int i = crank * kTkThreads + tid; i < n; i += CS * kTkThreads) {
      if (i < k) out[i] = i < L ? i : -1;
      rm.put(row, b, i, i < L ? i : -1, pc);
    }
    return;
  }


  const int slice = ceil_div(ceil_div(L, CS), kTkThreads) * kTkThreads;  // <= kTkSlice by launch
  const int s0 = crank * slice;
  const int lim = max(0, min(slice, L - s0));                 // valid elements of this slice
  const int nvalid = max(0, min(kTkPerThread, lim - tid * kTkPerThread));  // in this thread's chunk
  const int32_t* src = scores + (size_t)row * max_seqlen;

  // ---- load this CTA's slice (coalesced), keep keys in padded per-thread chunks ----
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int j = 0; j < kTkPerThread; ++j) {
    const int e = j * kTkThreads + tid;           // element within the slice
    uint32_t u = 0u;                               // past the slice: never read again
    if (e < lim) {
      u = static_cast<uint32_t>(src[s0 + e]) ^ 0x80000000u;
      kmin = min(kmin, u);
      kmax = max(kmax, u);
    }
    sm.keys[(e / kTkPerThread) * kTkChunkStride + (e % kTkPerThread)] = u;
  }
  if (hint != nullptr)
    for (int i = tid; i < kTkThreads * PER / 32; i += kTkThreads) sm.mark[i] = 0u;
  kmin = tk_block_reduce(kmin, sm.red, false);
  kmax = tk_block_reduce(kmax, sm.red, true);
  if (tid == 0) {
    sm.cta_vals[0] = kmin;
    sm.cta_vals[1] = kmax;
  }
  cluster.sync();
  if (tid < 32) {
    uint32_t mn = 0xffffffffu, mx = 0u;
    if (tid < CS) {
      const uint32_t* rv = cluster.map_shared_rank(sm.cta_vals, tid);
      mn = rv[0];
      mx = rv[1];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (tid == 0) {
      sm.found[0] = mn;
      sm.found[1] = mx;
    }
  }
  __syncthreads();
  uint32_t gmin = sm.found[0], gmax = sm.found[1];
  uint32_t hi_cut = 0xffffffffu;              // keys above it are all selected
  uint32_t remaining0 = static_cast<uint32_t>(k);

  // ---- previous selection as a hint (exact for any hint) ----
  // P = the hint's distinct tokens below L. If |P| = k, the k-th largest key
  // T* is at least lo = min over P, and at most max(lo, hi) with hi = max over
  // the other tokens (if T* exceeded both, the top-k would be P itself and
  // T* = lo). So the radix passes only resolve [lo, max(lo, hi)], after
  // taking every key above that range.
  if (hint != nullptr) {
    const int32_t* hr = hint + (size_t)row * k;
    for (int i = crank * kTkThreads + tid; i < k; i += CS * kTkThreads) {
      const int t = hr[i];
      if (t >= 0 && t < L) {
        const int owner = t / slice, off = t - owner * slice;
        atomicOr(cluster.map_shared_rank(sm.mark, owner) + (off >> 5), 1u << (off & 31));
      }
    }
    cluster.sync();  // every hint bit is set
    uint32_t lo = 0xffffffffu, hi = 0u, np = 0u;
    {
      const uint32_t* chunk = sm.keys + tid * kTkChunkStride;
      for (int j = 0; j < nvalid; ++j) {
        const int e = tid * kTkPerThread + j;
        const uint32_t u = chunk[j];
        if ((sm.mark[e >> 5] >> (e & 31)) & 1u) {
          lo = min(lo, u);
          ++np;
        } else {
          hi = max(hi, u);
        }
      }
    }
    lo = tk_block_reduce(lo, sm.red, false);
    hi = tk_block_reduce(hi, sm.red, true);
    uint32_t np_tot;
    tk_block_excl_scan(np, sm.red, &np_tot);
    if (tid == 0) {
      sm.hvals[0] = lo;
      sm.hvals[1] = hi;
      sm.hvals[2] = np_tot;
    }
    cluster.sync();
    if (tid < 32) {
      uint32_t l = 0xffffffffu, h = 0u, n = 0u;
      if (tid < CS) {
        const uint32_t* rv = cluster.map_shared_rank(sm.hvals, tid);
        l = rv[0];
        h = rv[1];
        n = rv[2];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        l = min(l, __shfl_xor_sync(0xffffffffu, l, o));
        h = max(h, __shfl_xor_sync(0xffffffffu, h, o));
        n += __shfl_xor_sync(0xffffffffu, n, o);
      }
      if (tid == 0) {
        sm.found[0] = l;
        sm.found[1] = n >= static_cast<uint32_t>(k) ? max(h, l) : 0xffffffffu;  // 0xffffffff: no bound
      }
    }
    __syncthreads();
    const uint32_t lo_all = sm.found[0], x = sm.found[1];
    __syncthreads();
    // narrow only when it saves a radix pass (the count above x costs one
    // cluster round trip); bound-less hints fall through to the full range
    auto passes = [](uint32_t a, uint32_t c) { return a == c ? 0 : (32 - __clz(a ^ c) + kTkBinsBits - 1) / kTkBinsBits; };
    if (x != 0xffffffffu && passes(lo_all, x) < passes(gmin, gmax)) {
      uint32_t above = 0u;
      const uint32_t* chunk = sm.keys + tid * kTkChunkStride;
      for (int j = 0; j < nvalid; ++j) above += chunk[j] > x;
      uint32_t above_cta;
      tk_block_excl_scan(above, sm.red, &above_cta);
      if (tid == 0) sm.hvals[3] = above_cta;
      cluster.sync();
      if (tid < 32) {
        uint32_t n = tid < CS ? cluster.map_shared_rank(sm.hvals, tid)[3] : 0u;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
        if (tid == 0) sm.found[0] = n;
      }
      __syncthreads();
      remaining0 = static_cast<uint32_t>(k) - sm.found[0];
      gmin = lo_all;
      gmax = x;
      hi_cut = x;
      __syncthreads();
    }
  }

  // ---- radix passes from the highest differing bit ----
  uint32_t T;                 // threshold key
  uint32_t need_eq;           // keys == T to take (in token order)
  if (gmin == gmax) {
    T = gmax;
    need_eq = remaining0;
  } else {
    const int hb = 31 - __clz(gmin ^ gmax);       // highest differing bit
    uint32_t prefix = hb == 31 ? 0u : (gmax >> (hb + 1)) << (hb + 1);
    uint32_t pmask = hb == 31 ? 0u : ~((2u << hb) - 1u);
    uint32_t remaining = remaining0;
    int top = hb;                                   // highest unresolved bit
    bool settled = false;
    T = 0;
    need_eq = 0;
    while (!settled) {
      const int nbits = min(kTkBinsBits, top + 1);
      const int shift = top + 1 - nbits;
      const uint32_t dmask = (1u << nbits) - 1u;
      for (int i = tid; i < kTkBins; i += kTkThreads) sm.hist[i] = 0u;
      __syncthreads();
      const uint32_t* chunk = sm.keys + tid * kTkChunkStride;
      for (int j = 0; j < nvalid; ++j) {
        const uint32_t u = chunk[j];
        if ((u & pmask) == prefix && u <= hi_cut) atomicAdd(&sm.hist[(u >> shift) & dmask], 1u);
      }
      cluster.sync();  // every CTA's histogram is complete
      for (int i = tid; i < kTkBins; i += kTkThreads) {
        uint32_t v = 0;
        for (int r = 0; r < CS; ++r) v += cluster.map_shared_rank(sm.hist, r)[i];
        sm.total[i] = v;
      }
      cluster.sync();  // nobody rewrites its histogram before all have read it
      // thread t owns bins 4t..4t+3; find the digit where the count of keys with
      // a larger-or-equal digit first reaches `remaining`
      uint32_t c4[4], mine = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        c4[i] = sm.total[4 * tid + i];
        mine += c4[i];
      }
      uint32_t all;
      // exclusive scan in reverse thread order = count of keys in higher bins
      const uint32_t rev = tk_block_excl_scan(mine, sm.red, &all);
      const uint32_t above = all - rev - mine;
      if (above < remaining && above + mine >= remaining) {
        uint32_t acc = above;
#pragma unroll
        for (int i = 3; i >= 0; --i) {
          if (acc < remaining && acc + c4[i] >= remaining) {
            sm.found[0] = 4u * tid + i;
            sm.found[1] = remaining - acc;
          }
          acc += c4[i];
        }
      }
      __syncthreads();
      const uint32_t digit = sm.found[0];
      const uint32_t rem = sm.found[1];
      const uint32_t bin_count = sm.total[digit];
      __syncthreads();
      prefix |= digit << shift;
      pmask |= dmask << shift;
      top = shift - 1;
      if (shift == 0) {            // every bit fixed: T is exact
        T = prefix;
        need_eq = rem;
        settled = true;
      } else if (bin_count == rem) {  // the whole bin is taken
        T = prefix;                // lowest key of the bin; all keys >= T are in
        need_eq = 0xffffffffu;
        settled = true;
      } else {
        remaining = rem;
      }
    }
  }

  // ---- ordered compaction ----
  const uint32_t* chunk = sm.keys + tid * kTkChunkStride;
  uint32_t n_gt = 0, n_eq = 0;
  for (int j = 0; j < nvalid; ++j) {
    const uint32_t u = chunk[j];
    n_gt += u > T;
    n_eq += u == T;
  }
  uint32_t tot_packed;
  const uint32_t pre = tk_block_excl_scan((n_gt << 16) | n_eq, sm.red, &tot_packed);
  if (tid == 0) {
    sm.cta_vals[2] = tot_packed >> 16;
    sm.cta_vals[3] = tot_packed & 0xffffu;
  }
  cluster.sync();
  uint32_t base_gt = 0, base_eq = 0;
  for (int r = 0; r < crank; ++r) {
    const uint32_t* rv = cluster.map_shared_rank(sm.cta_vals, r);
    base_gt += rv[2];
    base_eq += rv[3];
  }
  uint32_t gt_before = base_gt + (pre >> 16);
  uint32_t eq_before = base_eq + (pre & 0xffffu);
  for (int j = 0; j < nvalid; ++j) {
    const uint32_t u = chunk[j];
    const int g = s0 + tid * kTkPerThread + j;
    if (u > T) {
      out[gt_before + min(eq_before, need_eq)] = g;
      ++gt_before;
    } else if (u == T) {
      if (eq_before < need_eq) out[gt_before + eq_before] = g;
      ++eq_before;
    }
  }
  cluster.sync();  // no CTA leaves while others may still read its shared memory
  // optional row ids: a separate pass over the finished output (written by
  // the whole cluster before the barrier), one block-table load per page run
  if (rm.rows != nullptr)
    for (int i = crank * kTkThreads + tid; i < rm.kpad; i += CS * kTkThreads) rm.put(row, b, i, i < k ? out[i] : -1, pc);
}

// Cluster size for rows of up to max_seqlen scores with PER scores per thread
// (0: does not fit in kTkMaxCluster CTAs).
inline int topk_cluster_size(int max_seqlen, int per) {
  const long long slice = (long long)kTkThreads * per;
  int cs = 1;
  while (cs < kTkMaxCluster && cs * slice < max_seqlen) cs <<= 1;
  return cs * slice >= max_seqlen ? cs : 0;
}

}  // namespace sd
