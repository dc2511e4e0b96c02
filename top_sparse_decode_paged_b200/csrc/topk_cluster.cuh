// Per-row top-k of int32 indexer scores with one thread-block cluster per row.
//
// Same result as topk_radix_kernel (score descending, ties to the lower token,
// output in ascending token order, -1 padded), organised for B200:
//   - a row of L scores is split over a cluster of CS CTAs (CS <= 8); each CTA
//     copies its slice (NT = 1024 or 512 threads x 16 or 32 scores) once from L2 into shared
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
// Digit path (without a hint, the common case): the first radix pass fixes
// the digit D holding the k-th largest key (A keys above it, c_D in it). When
// c_D <= kTkDigitCap (a few dozen keys here), every CTA publishes its keys of
// D and its count above D, gathers the cluster's keys of D over DSMEM, ranks
// them to get the exact threshold, and writes its own slice's picks in token
// order: four cluster barriers in all, no pass over the full row after the
// first. When D holds more keys but A + c_D <= kTkCandCap, the candidate path
// has CTA 0 gather every key at or above D and resolve the threshold alone.
// Otherwise (heavy ties, or a hint) the radix passes run on the full slices
// as above.
// No CTA waits on another except at hardware cluster barriers.
#pragma once

#include <cooperative_groups.h>

#include "sd_common.cuh"

namespace sd {

namespace cg = cooperative_groups;

// NT: threads per CTA, 1024 (one CTA per SM: 32 warps keep the latency-bound
// phases busy) or 512 (two per SM, when that keeps every row in one wave).
constexpr int kTkMaxThreads = 1024;
constexpr int kTkBinsBits = 11;
constexpr int kTkBins = 1 << kTkBinsBits;
constexpr int kTkMaxCluster = 8;
constexpr int kTkCandCap = 4096;    // candidates (keys at or above the first pass's digit) the path takes
constexpr int kTkDigitCap = 512;    // keys of the threshold digit the digit path resolves in every CTA

// PER: scores per thread (16 or 32); a CTA holds a slice of NT * PER scores.
template <int PER, int NT>
struct TopkClusterSmem {
  static constexpr int kStride = PER + 1;       // padded per-thread chunk (words)
  uint32_t keys[NT * kStride];          // thread t's chunk at t*(PER+1) (bank-conflict free)
  uint32_t hist[kTkCandCap];                    // this CTA's histogram (read by the cluster); CTA 0's candidate keys
  uint32_t total[kTkCandCap];                   // cluster-wide histogram; CTA 0's candidate tokens
  uint32_t red[NT / 32 * 2 + 8];        // block reduction / scan scratch
  uint32_t cta_vals[4];                         // values this CTA publishes to the cluster
  uint32_t found[4];                            // threshold digit, remaining (and scratch)
  uint32_t mark[NT * PER / 32];         // hint tokens of this CTA's slice (one bit each)
  uint32_t hvals[4];                            // hint bounds this CTA publishes
  static_assert(NT * kStride >= 2 * kTkCandCap, "candidate keys and tokens fit in the key area");
};

// Block-wide exclusive scan of 32-bit values (NT <= 1024); returns the prefix,
// writes the total to *total.
template <int NT>
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
    const uint32_t w = lane < NT / 32 ? scratch[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    if (lane < NT / 32) scratch[lane] = wi - w;
    if (lane == 31) scratch[NT / 32] = wi;
  }
  __syncthreads();
  const uint32_t r = scratch[warp] + incl - v;
  *total = scratch[NT / 32];
  __syncthreads();
  return r;
}

// Block-wide minimum and maximum in one pass (two barriers).
template <int NT>
__device__ __forceinline__ void tk_block_minmax(uint32_t& mn, uint32_t& mx, uint32_t* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    scratch[2 * warp] = mn;
    scratch[2 * warp + 1] = mx;
  }
  __syncthreads();
  mn = 0xffffffffu;
  mx = 0u;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    mn = min(mn, scratch[2 * w]);
    mx = max(mx, scratch[2 * w + 1]);
  }
  __syncthreads();
}

template <int NT>
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
    v = lane < NT / 32 ? scratch[lane] : (is_max ? 0u : 0xffffffffu);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint32_t n = __shfl_xor_sync(0xffffffffu, v, o);
      v = is_max ? max(v, n) : min(v, n);
    }
    if (lane == 0) scratch[NT / 32] = v;
  }
  __syncthreads();
  v = scratch[NT / 32];
  __syncthreads();
  return v;
}

// total[i] = sum over the cluster's CTAs of hist[i] (2048 bins), with every
// remote read of a thread in flight together; ends with a block barrier.
template <int NT, typename Smem>
__device__ __forceinline__ void tk_merge_hist(Smem& sm, cg::cluster_group& cluster, int CS) {
  constexpr int kPer = kTkBins / NT;
  uint32_t v[kTkMaxCluster][kPer];
#pragma unroll
  for (int r = 0; r < kTkMaxCluster; ++r) {
    if (r < CS) {
      const uint32_t* h = cluster.map_shared_rank(sm.hist, r);
#pragma unroll
      for (int j = 0; j < kPer; ++j) v[r][j] = h[threadIdx.x + j * NT];
    }
  }
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    uint32_t t = 0;
#pragma unroll
    for (int r = 0; r < kTkMaxCluster; ++r)
      if (r < CS) t += v[r][j];
    sm.total[threadIdx.x + j * NT] = t;
  }
  __syncthreads();
}

// Finds the threshold digit of one radix pass: thread t owns the
// (kTkBins / NT) bins from (kTkBins / NT) * t of `h` (2048 bins); the digit is
// the bin where the count of keys in it and all higher bins first reaches
// `remaining`. Returns (digit, remaining within it) through found[0..1] and
// the count of the digit's bin through the return value.
template <int NT>
__device__ __forceinline__ uint32_t tk_find_digit(const uint32_t* h, uint32_t remaining, uint32_t* red,
                                                  uint32_t* found) {
  const int tid = threadIdx.x;
  uint32_t c[(kTkBins / NT)], mine = 0;
#pragma unroll
  for (int i = 0; i < (kTkBins / NT); ++i) {
    c[i] = h[(kTkBins / NT) * tid + i];
    mine += c[i];
  }
  uint32_t all;
  const uint32_t before = tk_block_excl_scan<NT>(mine, red, &all);  // keys in lower bins
  const uint32_t above = all - before - mine;                   // keys in higher bins
  if (above < remaining && above + mine >= remaining) {
    uint32_t acc = above;
#pragma unroll
    for (int i = (kTkBins / NT) - 1; i >= 0; --i) {
      if (acc < remaining && acc + c[i] >= remaining) {
        found[0] = static_cast<uint32_t>((kTkBins / NT) * tid + i);
        found[1] = remaining - acc;
      }
      acc += c[i];
    }
  }
  __syncthreads();
  const uint32_t bin_count = h[found[0]];
  return bin_count;
}

// The digit path (see the file comment): the first radix pass has fixed the
// digit D of the k-th largest key, whose keys are those with (u & pmask1) ==
// prefix1 (c_D <= kTkDigitCap of them over the cluster); `need` of them are
// to be taken. Every CTA publishes its keys of D (in token order) and its
// count of keys above D, gathers the cluster's keys of D (typically a few
// dozen), ranks them to find
// the exact threshold key Tk and how many keys equal to it to take, then
// writes its own slice's picks in token order at the offset the earlier
// CTAs' counts give.
template <int PER, int NT>
__device__ __forceinline__ void topk_digit_path(TopkClusterSmem<PER, NT>& sm, cg::cluster_group& cluster, int CS,
                                                int crank, int row, int b, int k, int s0, int nvalid,
                                                uint32_t prefix1, uint32_t pmask1, uint32_t need, int32_t* out,
                                                const RowMap& rm) {
  const int tid = threadIdx.x;
  const uint32_t hiD = prefix1 | ~pmask1;  // the largest key of digit D
  uint32_t* dkey = sm.total;                // this CTA's keys of D
  uint32_t* gkey = sm.total + kTkDigitCap;  // the cluster's keys of D
  const uint32_t* chunk = sm.keys + tid * (PER + 1);
  // 1. this CTA's counts above D and its keys of D
  uint32_t kv[PER];
  uint32_t n_above = 0, n_d = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    kv[j] = chunk[j];
    if (j < nvalid) {
      n_above += kv[j] > hiD;
      n_d += (kv[j] & pmask1) == prefix1;
    }
  }
  uint32_t tot;
  const uint32_t pre = tk_block_excl_scan<NT>((n_above << 16) | n_d, sm.red, &tot);
  uint32_t pos = pre & 0xffffu;
#pragma unroll
  for (int j = 0; j < PER; ++j)
    if (j < nvalid && (kv[j] & pmask1) == prefix1) dkey[pos++] = kv[j];
  if (tid == 0) {
    sm.cta_vals[2] = tot >> 16;
    sm.cta_vals[3] = tot & 0xffffu;
  }
  cluster.sync();  // every CTA's keys of D and counts are in place
  if (tid == 0) SD_PROBE_MARK(2, 9, 0);
  uint32_t a_r[kTkMaxCluster], d_r[kTkMaxCluster];
#pragma unroll
  for (int r = 0; r < kTkMaxCluster; ++r) {
    a_r[r] = 0u;
    d_r[r] = 0u;
    if (r < CS) {
      const uint32_t* rv = cluster.map_shared_rank(sm.cta_vals, r);
      a_r[r] = rv[2];
      d_r[r] = rv[3];
    }
  }
  uint32_t base_above = 0, base_d = 0, cD = 0;
#pragma unroll
  for (int r = 0; r < kTkMaxCluster; ++r) {
    base_above += r < crank ? a_r[r] : 0u;
    base_d += r < crank ? d_r[r] : 0u;
    cD += d_r[r];
  }
  {
    uint32_t off = 0;
#pragma unroll
    for (int r = 0; r < kTkMaxCluster; ++r) {
      if (r < CS) {
        const uint32_t* rk = cluster.map_shared_rank(dkey, r);
        for (uint32_t i = tid; i < d_r[r]; i += NT) gkey[off + i] = rk[i];
      }
      off += d_r[r];
    }
  }
  cluster.sync();  // every CTA has gathered: no more remote reads, any CTA may leave after this
  if (tid == 0) SD_PROBE_MARK(2, 10, 0);
  // 2. the exact threshold: key x of D is Tk when fewer than `need` keys of D
  // are above it and at least `need` are at or above it
  for (uint32_t i = tid; i < cD; i += NT) {
    const uint32_t x = gkey[i];
    uint32_t gt = 0, ge = 0;
    for (uint32_t q = 0; q < cD; ++q) {
      const uint32_t y = gkey[q];
      gt += y > x;
      ge += y >= x;
    }
    if (gt < need && need <= ge) {
      sm.found[0] = x;         // every such thread writes the same two values
      sm.found[1] = need - gt;
    }
  }
  __syncthreads();
  if (tid == 0) SD_PROBE_MARK(2, 11, 0);
  const uint32_t Tk = sm.found[0], need_eq = sm.found[1];
  // keys of D in earlier CTAs above / equal to Tk
  uint32_t gtD = 0, eqD = 0;
  for (uint32_t i = tid; i < base_d; i += NT) {
    gtD += gkey[i] > Tk;
    eqD += gkey[i] == Tk;
  }
  uint32_t tot2;
  tk_block_excl_scan<NT>((gtD << 16) | eqD, sm.red, &tot2);
  const uint32_t gt_base = base_above + (tot2 >> 16), eq_base = tot2 & 0xffffu;
  // 3. this slice's picks in token order: every key above Tk, then the first
  // need_eq keys equal to it over the cluster. They fill the output range
  // [o0, o0 + n_out) of this CTA; they are staged in shared memory, then the
  // indices and (in a decode step) the pool rows are written with every
  // block-table load of a thread in flight together.
  uint32_t n_gt = 0, n_eq = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    if (j < nvalid) {
      n_gt += kv[j] > Tk;
      n_eq += kv[j] == Tk;
    }
  }
  uint32_t tot3;
  const uint32_t pre3 = tk_block_excl_scan<NT>((n_gt << 16) | n_eq, sm.red, &tot3);
  const uint32_t o0 = gt_base + min(eq_base, need_eq);
  const uint32_t n_out = (tot3 >> 16) + min(eq_base + (tot3 & 0xffffu), need_eq) - min(eq_base, need_eq);
  uint32_t gt_before = gt_base + (pre3 >> 16), eq_before = eq_base + (pre3 & 0xffffu);
  uint32_t* stage = sm.hist;  // read by no CTA any more (the histogram merge is long done)
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    if (j < nvalid) {
      const uint32_t u = kv[j];
      const uint32_t g = static_cast<uint32_t>(s0 + tid * PER + j);
      if (u > Tk) {
        stage[gt_before + min(eq_before, need_eq) - o0] = g;
        ++gt_before;
      } else if (u == Tk) {
        if (eq_before < need_eq) stage[gt_before + eq_before - o0] = g;
        ++eq_before;
      }
    }
  }
  __syncthreads();
  if (tid == 0) SD_PROBE_MARK(2, 12, 0);
  constexpr int kOutPerThr = (kMaxTopK + NT - 1) / NT;
  int pages[kOutPerThr];
#pragma unroll
  for (int q = 0; q < kOutPerThr; ++q) {
    const uint32_t i = tid + q * NT;
    pages[q] = -1;
    if (i < n_out) {
      const int tok = static_cast<int>(stage[i]);
      out[o0 + i] = tok;
      if (rm.rows != nullptr) pages[q] = rm.block_table[(size_t)b * rm.max_pages + tok / rm.page_size];
    }
  }
  if (rm.rows != nullptr) {
#pragma unroll
    for (int q = 0; q < kOutPerThr; ++q) {
      const uint32_t i = tid + q * NT;
      if (i < n_out) rm.put_page(row, static_cast<int>(o0 + i), static_cast<int>(stage[i]), pages[q]);
    }
    if (crank == 0)
      for (int i = k + tid; i < rm.kpad; i += NT) rm.rows[(size_t)row * rm.kpad + i] = -1;
  }
  if (tid == 0) SD_PROBE_MARK(2, 5, cD);
}

// The candidate path (see the file comment). On entry the first radix pass
// has fixed the digit D of the k-th largest key: its keys are those with
// (u & pmask1) == prefix1 (bin_count of them, over the cluster), every key
// >= prefix1 is at or above D, and `need` keys are to be taken from D. Every
// CTA holds its slice's keys in its per-thread chunks. Ends with CTA 0
// writing the row's output; the other CTAs return after the third cluster
// barrier.
template <int PER, int NT>
__device__ __forceinline__ void topk_candidates(TopkClusterSmem<PER, NT>& sm, cg::cluster_group& cluster, int CS,
                                                int crank, int row, int b, int k, int s0, int nvalid,
                                                uint32_t prefix1, uint32_t pmask1, int shift, uint32_t need,
                                                uint32_t bin_count, int32_t* out, const RowMap& rm) {
  const int tid = threadIdx.x;
  // 1. this CTA's keys >= prefix1, in token order, into the key area
  uint32_t kv[PER];
  uint32_t pick = 0, nc = 0;
  const uint32_t* chunk = sm.keys + tid * (PER + 1);
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    kv[j] = chunk[j];
    const bool c = j < nvalid && kv[j] >= prefix1;
    pick |= static_cast<uint32_t>(c) << j;
    nc += c;
  }
  uint32_t ctot;
  uint32_t pos = tk_block_excl_scan<NT>(nc, sm.red, &ctot);  // its barriers order every chunk read before the writes
  uint32_t* ck = sm.keys;               // candidate keys, token order
  uint32_t* ct = sm.keys + kTkCandCap;  // their tokens
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    if ((pick >> j) & 1u) {
      ck[pos] = kv[j];
      ct[pos] = static_cast<uint32_t>(s0 + tid * PER + j);
      ++pos;
    }
  }
  if (tid == 0) sm.cta_vals[2] = ctot;
  cluster.sync();  // every CTA's candidates and count are in place (and every histogram read)
  uint32_t* gk = sm.hist;   // CTA 0: the cluster's candidates in token order (CTA slices are in order)
  uint32_t* gt = sm.total;
  if (crank == 0) {
    uint32_t cnt[kTkMaxCluster];
#pragma unroll
    for (int r = 0; r < kTkMaxCluster; ++r) cnt[r] = r < CS ? cluster.map_shared_rank(sm.cta_vals, r)[2] : 0u;
    uint32_t off = 0;
#pragma unroll
    for (int r = 0; r < kTkMaxCluster; ++r) {
      if (r < CS) {
        const uint32_t* rk = cluster.map_shared_rank(sm.keys, r);
        for (uint32_t i = tid; i < cnt[r]; i += NT) {
          gk[off + i] = rk[i];
          gt[off + i] = rk[kTkCandCap + i];
        }
      }
      off += cnt[r];
    }
    if (tid == 0) sm.found[0] = off;
  }
  cluster.sync();  // CTA 0 holds every candidate: the others may leave
  if (crank != 0) return;
  const uint32_t nC = sm.found[0];

  // 2. the exact threshold key Tk among the keys of digit D (radix passes over
  // the candidates, histogram in the now free key area)
  uint32_t Tk = prefix1, need_eq;
  if (shift == 0) {
    need_eq = need;                 // D is a single key value
  } else if (bin_count == need) {
    need_eq = 0xffffffffu;          // all of D is taken: every key >= prefix1 is in
  } else {
    uint32_t* rh = sm.keys;
    uint32_t prefix = prefix1, pmask = pmask1, remaining = need;
    int top = shift - 1;
    for (;;) {
      const int nbits = min(kTkBinsBits, top + 1);
      const int sh = top + 1 - nbits;
      const uint32_t dmask = (1u << nbits) - 1u;
      for (int i = tid; i < kTkBins; i += NT) rh[i] = 0u;
      __syncthreads();
      for (uint32_t i = tid; i < nC; i += NT) {
        const uint32_t u = gk[i];
        if ((u & pmask) == prefix) atomicAdd(&rh[(u >> sh) & dmask], 1u);
      }
      __syncthreads();
      const uint32_t cnt = tk_find_digit<NT>(rh, remaining, sm.red, sm.found + 2);
      const uint32_t digit = sm.found[2], rem = sm.found[3];
      __syncthreads();
      prefix |= digit << sh;
      pmask |= dmask << sh;
      top = sh - 1;
      if (sh == 0) {  // every bit fixed: Tk is exact
        Tk = prefix;
        need_eq = rem;
        break;
      }
      if (cnt == rem) {  // the whole digit bin is taken: every key >= prefix is in
        Tk = prefix;
        need_eq = 0xffffffffu;
        break;
      }
      remaining = rem;
    }
  }

  // 3. ordered output: candidate i is taken if its key is above Tk (every key
  // of a digit above D is), or equal to Tk and among the first need_eq of
  // those in token order; thread t handles kPerThr consecutive candidates
  constexpr int kPerThr = kTkCandCap / NT;
  uint32_t n_gt = 0, n_eq = 0;
#pragma unroll
  for (int j = 0; j < kPerThr; ++j) {
    const uint32_t i = kPerThr * tid + j;
    if (i < nC) {
      const uint32_t u = gk[i];
      n_gt += u > Tk;
      n_eq += u == Tk;
    }
  }
  uint32_t tot_packed;
  const uint32_t pre = tk_block_excl_scan<NT>((n_gt << 16) | n_eq, sm.red, &tot_packed);
  uint32_t gt_before = pre >> 16, eq_before = pre & 0xffffu;
  if (tid == 0) SD_PROBE_MARK(2, 3, nC);
  // the taken tokens in output order, staged in the free key area (k <= 2048)
  uint32_t* sel = sm.keys;
#pragma unroll
  for (int j = 0; j < kPerThr; ++j) {
    const uint32_t i = kPerThr * tid + j;
    if (i < nC) {
      const uint32_t u = gk[i];
      if (u > Tk) {
        sel[gt_before + min(eq_before, need_eq)] = gt[i];
        ++gt_before;
      } else if (u == Tk) {
        if (eq_before < need_eq) sel[gt_before + eq_before] = gt[i];
        ++eq_before;
      }
    }
  }
  __syncthreads();
  // coalesced output; the pool rows' block-table loads of a thread are
  // independent of each other, so they are all in flight together
  constexpr int kOutPerThr = (kMaxTopK + NT - 1) / NT;
  int pages[kOutPerThr];
#pragma unroll
  for (int j = 0; j < kOutPerThr; ++j) {
    const int o = tid + j * NT;
    pages[j] = -1;
    if (o < k) {
      const int tok = static_cast<int>(sel[o]);
      out[o] = tok;
      if (rm.rows != nullptr) pages[j] = rm.block_table[(size_t)b * rm.max_pages + tok / rm.page_size];
    }
  }
  if (rm.rows != nullptr) {
#pragma unroll
    for (int j = 0; j < kOutPerThr; ++j) {
      const int o = tid + j * NT;
      if (o < k) rm.put_page(row, o, static_cast<int>(sel[o]), pages[j]);
    }
    for (int i = k + tid; i < rm.kpad; i += NT) rm.rows[(size_t)row * rm.kpad + i] = -1;
  }
  if (tid == 0) SD_PROBE_MARK(2, 5, nC);
}

template <int PER, int NT>
__global__ void __launch_bounds__(NT, kTkMaxThreads / NT) topk_cluster_kernel(
    const int32_t* __restrict__ scores, const int32_t* __restrict__ seqlens, int32_t* __restrict__ indices,
    int G, int max_seqlen, int seqlen_cap, int k, RowMap rm, const int32_t* __restrict__ hint) {
  pdl_wait();  // inputs come from earlier work in the stream
  pdl_trigger();
  if (threadIdx.x == 0) SD_PROBE_MARK(2, 0, 0);

  constexpr int kTkPerThread = PER;
  constexpr int kTkChunkStride = PER + 1;
  extern __shared__ __align__(16) uint8_t tk_smem_raw[];
  TopkClusterSmem<PER, NT>& sm = *reinterpret_cast<TopkClusterSmem<PER, NT>*>(tk_smem_raw);
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
    for (int i = crank * NT + tid; i < n; i += CS * NT) {
      if (i < k) out[i] = i < L ? i : -1;
      rm.put(row, b, i, i < L ? i : -1, pc);
    }
    return;
  }


  const int slice = ceil_div(ceil_div(L, CS), NT) * NT;  // <= kTkSlice by launch
  const int s0 = crank * slice;
  const int lim = max(0, min(slice, L - s0));                 // valid elements of this slice
  const int nvalid = max(0, min(kTkPerThread, lim - tid * kTkPerThread));  // in this thread's chunk
  const int32_t* src = scores + (size_t)row * max_seqlen;

  // ---- load this CTA's slice (coalesced), keep keys in padded per-thread chunks ----
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int j = 0; j < kTkPerThread; ++j) {
    const int e = j * NT + tid;           // element within the slice
    uint32_t u = 0u;                               // past the slice: never read again
    if (e < lim) {
      u = static_cast<uint32_t>(src[s0 + e]) ^ 0x80000000u;
      kmin = min(kmin, u);
      kmax = max(kmax, u);
    }
    sm.keys[(e / kTkPerThread) * kTkChunkStride + (e % kTkPerThread)] = u;
  }
  if (hint != nullptr)
    for (int i = tid; i < NT * PER / 32; i += NT) sm.mark[i] = 0u;
  if (tid == 0) SD_PROBE_MARK(2, 6, 0);
  tk_block_minmax<NT>(kmin, kmax, sm.red);
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
  if (threadIdx.x == 0) SD_PROBE_MARK(2, 1, 0);
  uint32_t gmin = sm.found[0], gmax = sm.found[1];
  uint32_t hi_cut = 0xffffffffu;              // keys above it are all selected
  uint32_t remaining0 = static_cast<uint32_t>(k);

  // ---- candidate path: first radix pass, then one candidate exchange ----
  if (hint == nullptr && gmin != gmax) {
    const int hb = 31 - __clz(gmin ^ gmax);
    const uint32_t prefix0 = hb == 31 ? 0u : (gmax >> (hb + 1)) << (hb + 1);
    const uint32_t pmask0 = hb == 31 ? 0u : ~((2u << hb) - 1u);
    const int nbits = min(kTkBinsBits, hb + 1);
    const int shift = hb + 1 - nbits;
    const uint32_t dmask = (1u << nbits) - 1u;
    for (int i = tid; i < kTkBins; i += NT) sm.hist[i] = 0u;
    __syncthreads();
    {
      const uint32_t* chunk = sm.keys + tid * kTkChunkStride;
      for (int j = 0; j < nvalid; ++j) atomicAdd(&sm.hist[(chunk[j] >> shift) & dmask], 1u);
    }
    if (tid == 0) SD_PROBE_MARK(2, 7, 0);
    cluster.sync();  // every CTA's histogram is complete
    tk_merge_hist<NT>(sm, cluster, CS);
    if (tid == 0) SD_PROBE_MARK(2, 8, 0);
    const uint32_t bin_count = tk_find_digit<NT>(sm.total, static_cast<uint32_t>(k), sm.red, sm.found + 2);
    const uint32_t digit = sm.found[2], rem = sm.found[3];
    __syncthreads();
    const uint32_t above = static_cast<uint32_t>(k) - rem;
    const uint32_t prefix1 = prefix0 | (digit << shift), pmask1 = pmask0 | (dmask << shift);
    if (bin_count <= static_cast<uint32_t>(kTkDigitCap)) {
      if (threadIdx.x == 0) SD_PROBE_MARK(2, 2, bin_count);
      topk_digit_path<PER, NT>(sm, cluster, CS, crank, row, b, k, s0, nvalid, prefix1, pmask1, rem, out, rm);
      return;
    }
    if (above + bin_count <= static_cast<uint32_t>(kTkCandCap)) {
      if (threadIdx.x == 0) SD_PROBE_MARK(2, 2, bin_count);
      topk_candidates<PER, NT>(sm, cluster, CS, crank, row, b, k, s0, nvalid, prefix1, pmask1, shift, rem,
                           bin_count, out, rm);
      return;
    }
    // the full passes below start over and rewrite this CTA's histogram:
    // first let every CTA finish reading it
    cluster.sync();
  }

  // ---- previous selection as a hint (exact for any hint) ----
  // P = the hint's distinct tokens below L. If |P| = k, the k-th largest key
  // T* is at least lo = min over P, and at most max(lo, hi) with hi = max over
  // the other tokens (if T* exceeded both, the top-k would be P itself and
  // T* = lo). So the radix passes only resolve [lo, max(lo, hi)], after
  // taking every key above that range.
  if (hint != nullptr) {
    const int32_t* hr = hint + (size_t)row * k;
    for (int i = crank * NT + tid; i < k; i += CS * NT) {
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
    lo = tk_block_reduce<NT>(lo, sm.red, false);
    hi = tk_block_reduce<NT>(hi, sm.red, true);
    uint32_t np_tot;
    tk_block_excl_scan<NT>(np, sm.red, &np_tot);
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
      tk_block_excl_scan<NT>(above, sm.red, &above_cta);
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
      for (int i = tid; i < kTkBins; i += NT) sm.hist[i] = 0u;
      __syncthreads();
      const uint32_t* chunk = sm.keys + tid * kTkChunkStride;
      for (int j = 0; j < nvalid; ++j) {
        const uint32_t u = chunk[j];
        if ((u & pmask) == prefix && u <= hi_cut) atomicAdd(&sm.hist[(u >> shift) & dmask], 1u);
      }
      cluster.sync();  // every CTA's histogram is complete
      tk_merge_hist<NT>(sm, cluster, CS);
      cluster.sync();  // nobody rewrites its histogram before all have read it
      // the digit where the count of keys with a larger-or-equal digit first
      // reaches `remaining`
      const uint32_t bin_count = tk_find_digit<NT>(sm.total, remaining, sm.red, sm.found);
      const uint32_t digit = sm.found[0];
      const uint32_t rem = sm.found[1];
      __syncthreads();
      prefix |= digit << shift;
      pmask |= dmask << shift;
      top = shift - 1;
      if (threadIdx.x == 0) SD_PROBE_MARK(2, 2, bin_count);
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
  const uint32_t pre = tk_block_excl_scan<NT>((n_gt << 16) | n_eq, sm.red, &tot_packed);
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
  if (threadIdx.x == 0) SD_PROBE_MARK(2, 3, 0);
  cluster.sync();  // no CTA leaves while others may still read its shared memory
  // optional row ids: a separate pass over the finished output (written by
  // the whole cluster before the barrier), one block-table load per page run
  if (rm.rows != nullptr)
    for (int i = crank * NT + tid; i < rm.kpad; i += CS * NT) rm.put(row, b, i, i < k ? out[i] : -1, pc);
  if (threadIdx.x == 0) SD_PROBE_MARK(2, 4, 0);
}

// Cluster size for rows of up to max_seqlen scores with PER scores per thread
// (0: does not fit in kTkMaxCluster CTAs).
inline int topk_cluster_size(int max_seqlen, int per, int nt) {
  const long long slice = (long long)nt * per;
  int cs = 1;
  while (cs < kTkMaxCluster && cs * slice < max_seqlen) cs <<= 1;
  return cs * slice >= max_seqlen ? cs : 0;
}

}  // namespace sd
