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
//   z[b,h,p] = q_cal[h] . K[t, g]     fp32, products and sums in index order,
//                                     no fused multiply-add (reproducible)
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
// selection.
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

// Packed fp32 pair arithmetic: two independent IEEE round-to-nearest
// operations per instruction (no fusion, no flush to zero).
__device__ __forceinline__ unsigned long long tri_pack(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void tri_unpack(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long tri_mul2(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ unsigned long long tri_add2(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

constexpr int kTriStages = 3;

template <int D, int QPK>
struct TriScoreSmem {
  static constexpr int kStride = D * 2 + 16;  // padded row: per-thread row reads do not share banks
  uint8_t k[kTriStages][kTriThreads * kStride];
  float q[kTriStages][D * QPK];
  float wmax[kTriThreads / 32][QPK];
};

// z[b][h][p] and the per-tile maxima tmax[b][h][tile], one tile = 128
// consecutive evictable positions of one (request, KV head). Persistent: a
// CTA walks tiles blockIdx.x, + gridDim.x, ... through a 3-stage cp.async ring,
// so the rows of the next two tiles are in flight while a tile is summed.
// Thread r copies and sums row r of each tile (the row's page id is fetched
// one tile ahead into a register); a stage also holds the tile's q_cal slice,
// interleaved by head ([d][j]), so one broadcast load feeds every head at a
// given d. Each row is summed over d in index order, two heads per packed
// instruction.
template <int D, int QPK>
__global__ void __launch_bounds__(kTriThreads) tri_score_kernel(
    const float* __restrict__ q_cal, const __nv_bfloat16* __restrict__ k_pages, const int32_t* __restrict__ block_table,
    const int32_t* __restrict__ seqlens, int B, int H, int G, int page_size, int max_pages, int num_pages,
    int seqlen_cap, int n_sink, int n_recent, int e_max, float* __restrict__ z, float* __restrict__ tmax) {
  using Smem = TriScoreSmem<D, QPK>;
  constexpr int kChunks = D / 8, kStride = Smem::kStride;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  pdl_wait();  // every input may come from earlier work in the stream
  pdl_trigger();
  const int n_tiles = (e_max + kTriThreads - 1) / kTriThreads;
  const long long total = (long long)B * G * n_tiles;
  const int r = threadIdx.x;
  // tile k of this CTA: index blockIdx.x + k * gridDim.x
  auto tile_of = [&](int k, int& b, int& g, int& p0, int& E) -> bool {
    const long long T = blockIdx.x + (long long)k * gridDim.x;
    if (T >= total) return false;
    const int bg = static_cast<int>(T / n_tiles);
    b = bg / G;
    g = bg % G;
    p0 = static_cast<int>(T % n_tiles) * kTriThreads;
    E = tri_evictable(checked_seqlen(seqlens, b, seqlen_cap), n_sink, n_recent);
    return p0 < E;
  };
  auto page_of = [&](int k) -> int {  // row r's page in tile k (-1: no row)
    int b, g, p0, E;
    if (!tile_of(k, b, g, p0, E) || p0 + r >= E) return -1;
    const int t = n_sink + p0 + r;
    return block_table[(size_t)b * max_pages + t / page_size];
  };
  auto issue = [&](int k, int page) {  // tile k into stage k % kTriStages
    int b, g, p0, E;
    if (tile_of(k, b, g, p0, E)) {
      const int st = k % kTriStages;
      for (int i = r; i < D * QPK; i += kTriThreads) {  // q slice in [d][j] order
        const int d = i / QPK, j = i % QPK;
        cp_async_4(&sm.q[st][i], q_cal + (size_t)(g * QPK + j) * D + d);
      }
      const bool ok = p0 + r < E && page >= 0 && page < num_pages;
      const int t = n_sink + p0 + r;
      const uint8_t* src = reinterpret_cast<const uint8_t*>(
          k_pages + (((size_t)(ok ? page : 0) * page_size + t % page_size) * G + g) * D);
#pragma unroll
      for (int c = 0; c < kChunks; ++c) cp_async_16(&sm.k[st][r * kStride + c * 16], src + c * 16, ok ? 16 : 0);
    }
    cp_async_commit();  // one group per tile, empty or not
  };
  int pg_next = page_of(kTriStages - 1);
  for (int k = 0; k < kTriStages - 1; ++k) issue(k, page_of(k));
  for (int k = 0;; ++k) {
    int b, g, p0, E;
    const long long T = blockIdx.x + (long long)k * gridDim.x;
    if (T >= total) break;
    cp_async_wait<kTriStages - 2>();  // tile k has landed
    __syncthreads();                  // ... for every thread; stage (k - 1) % kTriStages is free
    issue(k + kTriStages - 1, pg_next);
    pg_next = page_of(k + kTriStages);
    if (!tile_of(k, b, g, p0, E)) continue;
    const int st = k % kTriStages;
    const bool in = p0 + r < E;
    int page = -1;
    if (in) page = block_table[(size_t)b * max_pages + (n_sink + p0 + r) / page_size];
    const bool live = in && page >= 0 && page < num_pages;
    if (in && !live) raise_error(SD_DEVERR_PAGE);
    const uint8_t* krow = &sm.k[st][r * kStride];
    const float* qs = sm.q[st];
    float zv[QPK];
    if constexpr (QPK == 1) {
      float acc = 0.f;
#pragma unroll 4
      for (int c = 0; c < kChunks; ++c) {
        const uint4 raw = *reinterpret_cast<const uint4*>(krow + c * 16);
        const __nv_bfloat16* kv = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
        for (int dd = 0; dd < 8; ++dd) acc = __fadd_rn(acc, __fmul_rn(qs[c * 8 + dd], __bfloat162float(kv[dd])));
      }
      zv[0] = acc;
    } else {
      constexpr int kPairs = QPK / 2;
      unsigned long long acc[kPairs];
#pragma unroll
      for (int j = 0; j < kPairs; ++j) acc[j] = 0ull;  // (+0.0f, +0.0f)
#pragma unroll 2
      for (int c = 0; c < kChunks; ++c) {
        const uint4 raw = *reinterpret_cast<const uint4*>(krow + c * 16);
        const __nv_bfloat16* kv = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
        for (int dd = 0; dd < 8; ++dd) {
          const float kf = __bfloat162float(kv[dd]);
          const unsigned long long kk = tri_pack(kf, kf);
          unsigned long long qp[kPairs];
          if constexpr (QPK == 2) {
            qp[0] = *reinterpret_cast<const unsigned long long*>(qs + (c * 8 + dd) * QPK);
          } else {
#pragma unroll
            for (int v = 0; v < QPK / 4; ++v) {
              const ulonglong2 q4 = *reinterpret_cast<const ulonglong2*>(qs + (c * 8 + dd) * QPK + 4 * v);
              qp[2 * v] = q4.x;
              qp[2 * v + 1] = q4.y;
            }
          }
#pragma unroll
          for (int j = 0; j < kPairs; ++j) acc[j] = tri_add2(acc[j], tri_mul2(qp[j], kk));
        }
      }
#pragma unroll
      for (int j = 0; j < kPairs; ++j) tri_unpack(acc[j], zv[2 * j], zv[2 * j + 1]);
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
      if ((r & 31) == 0) sm.wmax[r >> 5][j] = m;
    }
    __syncthreads();
    if (r < QPK) {
      float m = sm.wmax[0][r];
#pragma unroll
      for (int w = 1; w < kTriThreads / 32; ++w) m = fmaxf(m, sm.wmax[w][r]);
      tmax[((size_t)b * H + g * QPK + r) * n_tiles + p0 / kTriThreads] = m;
    }
  }
  cp_async_wait<0>();  // no copy may outlive the CTA
}

constexpr int kTriReduceThreads = 256;
constexpr int kTriMaxHeads = 256;

// Selection keys: one block per (256 positions, selection row). The per-head
// maxima come from the score tiles' maxima (one warp per head); a row's score
// at p is the maximum over its heads of z - m. Also zeroes the row's
// compaction flags.
__global__ void __launch_bounds__(kTriReduceThreads) tri_reduce_kernel(
    const float* __restrict__ z, const float* __restrict__ tmax, const int32_t* __restrict__ seqlens, int H, int G,
    int rows_per_req, int seqlen_cap, int n_sink, int n_recent, int e_max, int32_t* __restrict__ keys,
    int32_t* __restrict__ evictable, int32_t* __restrict__ flags, int n_chunks) {
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
  const int n_tiles = (e_max + kTriThreads - 1) / kTriThreads;
  const int live_tiles = (E + kTriThreads - 1) / kTriThreads;
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
  keys[(size_t)r * e_max + p] = tri_key(s);
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
constexpr int kTriChunkBytes = 32768;                 // K + V bytes of one unit
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
// (source == destination) are skipped. A wait that runs out sets
// SD_DEVERR_TIMEOUT and skips that unit's writes.
__global__ void __launch_bounds__(kTriCompactThreads) tri_compact_kernel(
    uint8_t* __restrict__ k_pages, uint8_t* __restrict__ v_pages, const int32_t* __restrict__ block_table,
    const int32_t* __restrict__ seqlens, const int32_t* __restrict__ sel, int rows_per_req, int page_size,
    int max_pages, int num_pages, int seqlen_cap, int n_sink, int n_recent, int budget, int part, int row_bytes,
    int chunk, int n_chunks, int n_rows, int32_t* __restrict__ flags, int32_t* __restrict__ new_seqlens) {
  pdl_wait();
  __shared__ __align__(16) uint8_t buf[kTriChunkBytes];
  __shared__ long long src_off[kTriMaxChunkTokens], dst_off[kTriMaxChunkTokens];
  __shared__ int wait_lo, wait_hi, wait_ok, search[2];
  const int moved = budget + n_recent;
  const int pieces_per_part = part / 16;
  const int pieces_per_token = pieces_per_part * (v_pages ? 2 : 1);
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
    // 1. sources into shared memory
    for (int pc = threadIdx.x; pc < nj * pieces_per_token; pc += kTriCompactThreads) {
      const int i = pc / pieces_per_token, w = pc % pieces_per_token;
      const long long so = src_off[i];
      if (so < 0) continue;
      const uint8_t* base = w < pieces_per_part ? k_pages : v_pages;
      cp_async_16(buf + pc * 16, base + so + (w % pieces_per_part) * 16, 16);
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
      for (; it < kTriWaitLimit; ++it) {
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
      for (int pc = threadIdx.x; pc < nj * pieces_per_token; pc += kTriCompactThreads) {
        const int i = pc / pieces_per_token, w = pc % pieces_per_token;
        const long long dof = dst_off[i];
        if (dof < 0) continue;
        uint8_t* base = w < pieces_per_part ? k_pages : v_pages;
        *reinterpret_cast<uint4*>(base + dof + (w % pieces_per_part) * 16) =
            *reinterpret_cast<const uint4*>(buf + pc * 16);
      }
    }
    __syncthreads();  // buf and the offsets are reused by the next unit
  }
}

}  // namespace sd
