// TriAttention-style decode-time eviction for one layer: score the evictable
// decode region of each request with calibrated per-head queries, keep the
// best `budget` tokens, and compact the kept K/V rows in place ("Add
// TriAttention KV-cache compression method", Summary and Key Design
// Decisions: paged-K scoring read in place, normalize/reduce, top-k with tie
// settlement, batched physical compaction, union / per-head modes).
//
// Scoring (a reading; the pages do not write the formula). For request b,
// query head h (KV head g = h * G / H) and evictable position p (token
// t = n_sink + p, p < E_b = L_b - n_sink - n_recent):
//   z[b,h,p] = q_cal[h] . K[t, g]     q_cal and K bf16, summed in fp32: one
//                                     fused multiply-add per d (the product is
//                                     exact; equal inputs give equal scores)
//   m[b,h]   = max_p z[b,h,p]
//   s[b,g,p] = max over the heads h of KV head g of (z[b,h,p] - m[b,h])
//   union:     s[b,p] = max_g s[b,g,p]
// Each head's logits are shifted to a common maximum of 0, so the heads are
// comparable; the maximum over heads keeps a token any head attends to.
// Selection: the `budget` largest scores, ties to the lower position (the
// library's top-k on an order-preserving integer image of the fp32 scores).
// Kept: the sink prefix [0, n_sink), the selected positions in order, then
// the recent tail [L - n_recent, L); the request's new length is
// n_sink + budget + n_recent. Requests with E_b <= budget keep everything.
// Compaction moves kept token i from logical position t_i to position i in
// one pass over the pools (see tri_compact_kernel). Union mode moves whole
// rows (all KV heads); per-head mode moves each KV head's part by its own
// selection. Selections shared across layers are composed on the host: the
// key pass folds each layer's scores in by maximum, then every layer is
// compacted with the one selection.
#pragma once

#include "sd_common.cuh"

namespace sd {

constexpr int kTriThreads = 128;

// Order-preserving int32 image of an fp32 score (for non-NaN values).
__device__ __forceinline__ int32_t tri_key(float f) {
  const int32_t i = __float_as_int(f);
  return i >= 0 ? i : (i ^ 0x7fffffff);
}

__device__ __forceinline__ int tri_evictable(int L, int n_sink, int n_recent) {
  return max(0, L - n_sink - n_recent);
}

constexpr int kTriTileTok = kTriThreads;  // evictable positions per score tile

// z[b][h][p] and the per-tile maxima tmax[b][h][tile] for one tile of 128
// consecutive evictable positions of one (request, KV head) per CTA. The
// tile's K rows (one D-wide bf16 segment per token) are staged in shared
// memory by coalesced 16-byte cp.async (kChunks lanes per row; rows padded by
// 16 bytes so that the per-thread row reads do not share banks); the KV
// head's q_cal slice sits there as fp32 in [d][j] order, so one broadcast
// load feeds four heads at a given d. Each row's source offset is computed
// once (no division per copied piece).
// Thread r sums row r over d in index order, one fused multiply-add per
// (d, head). Small CTAs (about 40 KB) let five share an SM, so copies of some
// overlap the arithmetic of others.
template <int D, int QPK>
__global__ void __launch_bounds__(kTriThreads) tri_score_kernel(
    const __nv_bfloat16* __restrict__ q_cal, const __nv_bfloat16* __restrict__ k_pages,
    const int32_t* __restrict__ block_table, const int32_t* __restrict__ seqlens, int H, int G, int page_size,
    int max_pages, int num_pages, int seqlen_cap, int n_sink, int n_recent, int e_max, float* __restrict__ z,
    float* __restrict__ tmax) {
  constexpr int kRowBytes = D * 2, kStride = kRowBytes + 16, kChunks = kRowBytes / 16;
  __shared__ __align__(16) uint8_t ks[kTriThreads * kStride];
  __shared__ __align__(16) float qs[D * QPK];
  __shared__ long long roff[kTriThreads];
  __shared__ float wmax[kTriThreads / 32][QPK];
  const int b = blockIdx.y / G, g = blockIdx.y % G;
  pdl_wait();  // every input may come from earlier work in the stream
  pdl_trigger();
  const int r = threadIdx.x;
  const int p0 = blockIdx.x * kTriTileTok;
  // independent loads first: the length, row r's block-table entry (read
  // whether or not the row exists, inside the request's table row) and this
  // thread's share of q_cal
  const int t = n_sink + p0 + r;
  const int pi = t / page_size;
  const int page_raw = pi < max_pages ? block_table[(size_t)b * max_pages + pi] : -1;
  float qv[(D * QPK + kTriThreads - 1) / kTriThreads];
#pragma unroll
  for (int m = 0; m < (D * QPK + kTriThreads - 1) / kTriThreads; ++m) {
    const int i = r + m * kTriThreads;
    qv[m] = i < D * QPK ? __bfloat162float(q_cal[(size_t)(g * QPK + i % QPK) * D + i / QPK]) : 0.f;
  }
  const int L = checked_seqlen(seqlens, b, seqlen_cap);
  const int E = tri_evictable(L, n_sink, n_recent);
  if (p0 >= E) return;
  const int nrows = min(kTriTileTok, E - p0);
  const bool in = r < nrows;
  // row r's source offset, once, for every copy of the row (-1: no row)
  long long off = -1;
  if (in) {
    if (page_raw >= 0 && page_raw < num_pages)
      off = (((long long)page_raw * page_size + t % page_size) * G + g) * kRowBytes;
    else
      raise_error(SD_DEVERR_PAGE);
  }
  const bool live = off >= 0;
  roff[r] = off;
#pragma unroll
  for (int m = 0; m < (D * QPK + kTriThreads - 1) / kTriThreads; ++m) {  // [d][j] <- q_cal[g * QPK + j][d]
    const int i = r + m * kTriThreads;
    if (i < D * QPK) qs[i] = qv[m];
  }
  __syncthreads();
  const uint8_t* kbase = reinterpret_cast<const uint8_t*>(k_pages);
#pragma unroll 4
  for (int i = threadIdx.x; i < nrows * kChunks; i += kTriThreads) {
    const int rr = i / kChunks, c = i % kChunks;  // kChunks is a power of two
    const long long o = roff[rr];
    cp_async_16(ks + rr * kStride + c * 16, kbase + (o >= 0 ? o : 0) + c * 16, o >= 0 ? 16 : 0);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  const uint8_t* krow = ks + r * kStride;
  float zv[QPK];
#pragma unroll
  for (int j = 0; j < QPK; ++j) zv[j] = 0.f;
#pragma unroll 2
  for (int c = 0; c < kChunks; ++c) {
    const uint4 raw = *reinterpret_cast<const uint4*>(krow + c * 16);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int dd = 0; dd < 8; ++dd) {
      // bf16 -> fp32: the 16 bits become the high half
      const float kf = __uint_as_float(dd & 1 ? (w[dd >> 1] & 0xffff0000u) : (w[dd >> 1] << 16));
      const float* qd = qs + (c * 8 + dd) * QPK;
      if constexpr (QPK % 4 == 0) {
#pragma unroll
        for (int v = 0; v < QPK / 4; ++v) {
          const float4 q4 = *reinterpret_cast<const float4*>(qd + 4 * v);
          zv[4 * v + 0] = __fmaf_rn(q4.x, kf, zv[4 * v + 0]);
          zv[4 * v + 1] = __fmaf_rn(q4.y, kf, zv[4 * v + 1]);
          zv[4 * v + 2] = __fmaf_rn(q4.z, kf, zv[4 * v + 2]);
          zv[4 * v + 3] = __fmaf_rn(q4.w, kf, zv[4 * v + 3]);
        }
      } else {
#pragma unroll
        for (int j = 0; j < QPK; ++j) zv[j] = __fmaf_rn(qd[j], kf, zv[j]);
      }
    }
  }
  // positions past the region and rows on a bad page count as -inf
#pragma unroll
  for (int j = 0; j < QPK; ++j) zv[j] = live ? zv[j] : -INFINITY;
  if (in) {
    float* zb = z + ((size_t)b * H + g * QPK) * e_max + p0 + r;
#pragma unroll
    for (int j = 0; j < QPK; ++j) zb[(size_t)j * e_max] = zv[j];
  }
  // this tile's maximum per query head, for the per-head shift
#pragma unroll
  for (int j = 0; j < QPK; ++j) {
    float m = zv[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((r & 31) == 0) wmax[r >> 5][j] = m;
  }
  __syncthreads();
  if (r < QPK) {
    float m = wmax[0][r];
#pragma unroll
    for (int w = 1; w < kTriThreads / 32; ++w) m = fmaxf(m, wmax[w][r]);
    const int n_tiles = (e_max + kTriTileTok - 1) / kTriTileTok;
    tmax[((size_t)b * H + g * QPK + r) * n_tiles + blockIdx.x] = m;
  }
}

constexpr int kTriReduceThreads = 256;
constexpr int kTriMaxHeads = 256;

// Selection keys: one block per (256 positions, selection row). The per-head
// maxima come from the score tiles' maxima (one warp per head); a row's score
// at p is the maximum over its heads of z - m, or, with `accumulate` (a later
// layer of a cross-layer selection), the maximum of that and the key already
// there. Also zeroes the row's compaction flags.
__global__ void __launch_bounds__(kTriReduceThreads) tri_reduce_kernel(
    const float* __restrict__ z, const float* __restrict__ tmax, const int32_t* __restrict__ seqlens, int H, int G,
    int rows_per_req, int seqlen_cap, int n_sink, int n_recent, int e_max, int32_t* __restrict__ keys,
    int32_t* __restrict__ evictable, int32_t* __restrict__ flags, int n_chunks, int accumulate) {
  pdl_wait();
  pdl_trigger();
  __shared__ float m_s[kTriMaxHeads];
  const int r = blockIdx.y;
  const int b = r / rows_per_req;
  const int qpk = H / G;
  const int h0 = rows_per_req == 1 ? 0 : (r % rows_per_req) * qpk;
  const int nh = rows_per_req == 1 ? H : qpk;
  for (int i = blockIdx.x * kTriReduceThreads + threadIdx.x; i < n_chunks; i += gridDim.x * kTriReduceThreads)
    flags[(size_t)r * n_chunks + i] = 0;
  const int L = checked_seqlen(seqlens, b, seqlen_cap);
  const int E = tri_evictable(L, n_sink, n_recent);
  if (blockIdx.x == 0 && threadIdx.x == 0 && (r % rows_per_req) == 0) evictable[b] = E;
  const int p0 = blockIdx.x * kTriReduceThreads;
  if (p0 >= E) return;
  const int n_tiles = (e_max + kTriTileTok - 1) / kTriTileTok;
  const int live_tiles = (E + kTriTileTok - 1) / kTriTileTok;
  const float* tb = tmax + ((size_t)b * H + h0) * n_tiles;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int h = warp; h < nh; h += kTriReduceThreads / 32) {
    float m = -INFINITY;
    for (int t = lane; t < live_tiles; t += 32) m = fmaxf(m, tb[(size_t)h * n_tiles + t]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) m_s[h] = m;
  }
  __syncthreads();
  const int p = p0 + threadIdx.x;
  if (p >= E) return;
  const float* zb = z + ((size_t)b * H + h0) * e_max + p;
  float s = -INFINITY;
  int h = 0;
  for (; h + 8 <= nh; h += 8) {
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = zb[(size_t)(h + i) * e_max];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (m_s[h + i] != -INFINITY) s = fmaxf(s, __fsub_rn(v[i], m_s[h + i]));
  }
  for (; h < nh; ++h)
    if (m_s[h] != -INFINITY) s = fmaxf(s, __fsub_rn(zb[(size_t)h * e_max], m_s[h]));
  int32_t* kp = keys + (size_t)r * e_max + p;
  const int32_t key = tri_key(s);
  *kp = accumulate ? max(*kp, key) : key;  // the key order is the score order
}

// Source of kept token j (0-based after the prefix) of a request.
__device__ __forceinline__ int tri_src(int j, int n_sink, int budget, int L, int n_recent,
                                       const int32_t* __restrict__ sel) {
  return j < budget ? n_sink + sel[j] : L - n_recent + (j - budget);
}

// First j in [0, n) with tri_src(j) >= x (n when none), by one warp: each
// step probes 32 evenly spaced j and keeps the gap where the predicate turns
// true (tri_src is increasing in j), so a range of n shrinks in log32(n) steps.
__device__ __forceinline__ int tri_warp_search(int x, int n, int n_sink, int budget, int L, int n_recent,
                                               const int32_t* __restrict__ sel) {
  const int lane = threadIdx.x & 31;
  int lo = 0, hi = n;  // the answer lies in [lo, hi]
  while (lo < hi) {
    const int step = (hi - lo + 31) / 32;
    const int pos = lo + lane * step;
    const bool ge = pos >= hi || tri_src(pos, n_sink, budget, L, n_recent, sel) >= x;
    const unsigned m = __ballot_sync(0xffffffffu, ge);
    if (m == 0) {
      lo = lo + 31 * step + 1;
    } else {
      const int f = __ffs(m) - 1;
      if (f == 0) {
        hi = lo;
      } else {
        const int new_lo = lo + (f - 1) * step + 1;
        hi = min(hi, lo + f * step);
        lo = new_lo;
      }
    }
  }
  return lo;
}

constexpr int kTriCompactThreads = 256;
constexpr int kTriChunkBytes = 32768;  // K + V bytes of one unit
constexpr int kTriMaxChunkTokens = kTriChunkBytes / 128;
constexpr uint32_t kTriWaitLimit = 1u << 22;

// One-pass in-place compaction. Kept token j moves from tri_src(j) to
// position n_sink + j, and tri_src(j) >= n_sink + j (the selection is
// ascending), so a token's destination is read only by kept tokens at or
// before it. Work is cut into units of `chunk` consecutive kept tokens of one
// selection row; a unit
//   1. copies its sources into shared memory (cp.async, completed) and
//      publishes flags[unit] = 1 (release);
//   2. finds by search (the source map is increasing; two warps, while the
//      copies are in flight) the kept tokens that read its destinations, and
//      waits (acquire, bounded) for the earlier units holding them;
//   3. writes its rows to their destinations.
// The grid is persistent (every CTA resident) and each CTA takes units in
// increasing order, so the smallest unfinished unit never waits on a unit
// that has not started; no dependent launch is triggered early, so no later
// kernel takes an SM slot while units wait. Tokens already in place
// (source == destination) are skipped. A wait gives up after `wait_limit`
// polls (kTriWaitLimit unless a test lowers it; 0 gives up at once): it sets
// SD_DEVERR_TIMEOUT and that unit skips its writes. No copy is in flight at
// that point (step 1 has completed), so the unit simply moves on.
__global__ void __launch_bounds__(kTriCompactThreads) tri_compact_kernel(
    uint8_t* __restrict__ k_pages, uint8_t* __restrict__ v_pages, const int32_t* __restrict__ block_table,
    const int32_t* __restrict__ seqlens, const int32_t* __restrict__ sel, int rows_per_req, int page_size,
    int max_pages, int num_pages, int seqlen_cap, int n_sink, int n_recent, int budget, int part, int row_bytes,
    int chunk, int n_chunks, int n_rows, int32_t* __restrict__ flags, int32_t* __restrict__ new_seqlens,
    uint32_t wait_limit) {
  pdl_wait();
  __shared__ __align__(16) uint8_t buf[kTriChunkBytes];
  __shared__ long long src_off[kTriMaxChunkTokens], dst_off[kTriMaxChunkTokens];
  __shared__ int wait_lo, wait_hi, wait_ok, search[2];
  const int moved = budget + n_recent;
  const int pieces_per_part = part / 16;
  const int pieces_per_token = pieces_per_part * (v_pages ? 2 : 1);
  const int step_i = kTriCompactThreads / pieces_per_token, step_w = kTriCompactThreads % pieces_per_token;
  const long long n_units = (long long)n_rows * n_chunks;
  for (long long u = blockIdx.x; u < n_units; u += gridDim.x) {
    const int r = static_cast<int>(u / n_chunks), c = static_cast<int>(u % n_chunks);
    const int b = r / rows_per_req, g = r % rows_per_req;
    const int L = checked_seqlen(seqlens, b, seqlen_cap);
    const int E = tri_evictable(L, n_sink, n_recent);
    if (c == 0 && g == 0 && threadIdx.x == 0) new_seqlens[b] = E <= budget ? L : n_sink + moved;
    if (E <= budget) continue;  // nothing evicted: no unit of this row moves anything
    const int32_t* srow = sel + (size_t)r * budget;
    const int j0 = c * chunk, nj = min(chunk, moved - j0);
    const int32_t* bt = block_table + (size_t)b * max_pages;
    for (int i = threadIdx.x; i < nj; i += kTriCompactThreads) {
      const int t = tri_src(j0 + i, n_sink, budget, L, n_recent, srow), d = n_sink + j0 + i;
      long long so = -1, dof = -1;
      if (t != d) {
        const int sp = bt[t / page_size], dp = bt[d / page_size];
        if (sp >= 0 && sp < num_pages && dp >= 0 && dp < num_pages) {
          so = ((long long)sp * page_size + t % page_size) * row_bytes + (long long)g * part;
          dof = ((long long)dp * page_size + d % page_size) * row_bytes + (long long)g * part;
        } else {
          raise_error(SD_DEVERR_PAGE);
        }
      }
      src_off[i] = so;
      dst_off[i] = dof;
    }
    __syncthreads();
    // 1. sources into shared memory (piece pc = token i, piece w of the token;
    // indices advance by carries, not by division)
    {
      int i = threadIdx.x / pieces_per_token, w = threadIdx.x % pieces_per_token;
      for (int pc = threadIdx.x; pc < nj * pieces_per_token; pc += kTriCompactThreads) {
        const long long so = src_off[i];
        if (so >= 0) {
          const bool kpart = w < pieces_per_part;
          cp_async_16(buf + pc * 16, (kpart ? k_pages : v_pages) + so + (kpart ? w : w - pieces_per_part) * 16, 16);
        }
        w += step_w;
        i += step_i;
        if (w >= pieces_per_token) {
          w -= pieces_per_token;
          ++i;
        }
      }
    }
    cp_async_commit();
    // while the copies fly: the kept tokens whose sources lie in
    // [n_sink + j0, n_sink + j0 + nj) are [first(j0), first(j0 + nj))
    if (threadIdx.x < 64) {
      const int x = n_sink + j0 + (threadIdx.x < 32 ? 0 : nj);
      const int j = tri_warp_search(x, moved, n_sink, budget, L, n_recent, srow);
      if ((threadIdx.x & 31) == 0) search[threadIdx.x >> 5] = j;
    }
    cp_async_wait<0>();
    __syncthreads();
    if (threadIdx.x == 0) {
      const int lo = search[0], lo2 = search[1];
      // chunks [wait_lo, wait_hi) hold those readers; this one is excluded
      wait_lo = lo / chunk;
      wait_hi = lo2 > lo ? min(c, (lo2 - 1) / chunk + 1) : wait_lo;
      wait_ok = 1;
    }
    if (threadIdx.x == 0) {
      __threadfence();
      asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(flags + u), "r"(1) : "memory");
    }
    __syncthreads();  // wait_lo / wait_hi
    // 2. wait for the earlier units that read this unit's destinations
    for (int cc = wait_lo + threadIdx.x; cc < wait_hi; cc += kTriCompactThreads) {
      const int32_t* f = flags + (size_t)r * n_chunks + cc;
      uint32_t it = 0;
      int v = 0;
      for (; it < wait_limit; ++it) {
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
        if (v) break;
        __nanosleep(64);
      }
      if (!v) {
        raise_error(SD_DEVERR_TIMEOUT);
        wait_ok = 0;
      }
    }
    __syncthreads();
    // 3. destinations
    if (wait_ok) {
      int i = threadIdx.x / pieces_per_token, w = threadIdx.x % pieces_per_token;
      for (int pc = threadIdx.x; pc < nj * pieces_per_token; pc += kTriCompactThreads) {
        const long long dof = dst_off[i];
        if (dof >= 0) {
          const bool kpart = w < pieces_per_part;
          *reinterpret_cast<uint4*>((kpart ? k_pages : v_pages) + dof + (kpart ? w : w - pieces_per_part) * 16) =
              *reinterpret_cast<const uint4*>(buf + pc * 16);
        }
        w += step_w;
        i += step_i;
        if (w >= pieces_per_token) {
          w -= pieces_per_token;
          ++i;
        }
      }
    }
    __syncthreads();  // buf and the offsets are reused by the next unit
  }
}

}  // namespace sd
