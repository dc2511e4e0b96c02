// Indexer scores on CUDA cores (dp4a), any supported (G, Hi, Di).
//
//   s[b,g,t] = sum_h w[b,g,h] * max(0, sum_d qi[b,g,h,d] * ki[t,g,d])
//
// Keys are read in place from the paged int8 pool through the block table
// (the pages' "direct paged-pool scoring ... no Torch gather" of the TriAttention
// scorer, Key Design Decisions). This kernel is the general path, for every
// shape the tensor-core kernel (indexer_umma.cuh) does not take: that one
// serves the MLA indexer (one KV head, Hi = 64, Di = 128) and the per-head
// indexer of 8 KV heads with Hi = 4, Di = 64.
//
// A CTA scores T consecutive tokens of one request for every KV head. Each
// token's row base is looked up once; the tile's key rows (G x Di bytes per
// token, contiguous in the pool) are then staged in shared memory by
// coalesced 16-byte cp.async, the 16-byte chunks XOR-swizzled so that
// per-thread row reads do not share banks. Threads then score (token, KV
// head) pairs from shared memory, q read from per-head blocks padded onto
// distinct banks. Indices advance by carries, not by division. T is chosen so
// that a tile takes about 32 KB, letting several CTAs share an SM.
#pragma once

#include "sd_common.cuh"

namespace sd {

constexpr int kIdxThreads = 256;
constexpr int kIdxTileBytes = 32768;  // key bytes per CTA

// Tokens per CTA for a key row of G * Di bytes per token.
__host__ __device__ inline int indexer_dp4a_tokens(int G, int Di) {
  const int t = kIdxTileBytes / (G * Di);
  return t < 1 ? 1 : (t > kIdxThreads ? kIdxThreads : t);
}

template <int DI>
__device__ __forceinline__ int idx_swz(int c, int row) {  // chunk c of row `row` in shared memory
  constexpr int kCpr = DI / 16;                   // 16-byte chunks per row
  constexpr int kRpl = DI >= 128 ? 1 : 128 / DI;  // rows per 128-byte line
  return c ^ ((row / kRpl) & (kCpr - 1));
}

template <int DI>
__global__ void __launch_bounds__(kIdxThreads) indexer_dp4a_kernel(
    const int8_t* __restrict__ qi, const int32_t* __restrict__ w, const int8_t* __restrict__ ki_pages,
    const int32_t* __restrict__ block_table, const int32_t* __restrict__ seqlens,
    int32_t* __restrict__ scores, int num_pages, int page_size, int max_pages, int G, int Hi,
    int max_seqlen) {
  pdl_wait();  // inputs come from earlier work in the stream
  pdl_trigger();

  constexpr int W4 = DI / 4;      // int32 words per key row
  constexpr int kCpr = DI / 16;   // 16-byte chunks per key row
  extern __shared__ __align__(16) int32_t smem_i32[];
  const int T = indexer_dp4a_tokens(G, DI);
  const int b = blockIdx.y;
  const int t0 = blockIdx.x * T;
  const int cap = min(max_seqlen, max_pages * page_size);
  const int L = checked_seqlen(seqlens, b, cap);
  if (t0 >= L) return;
  const int nt = min(L - t0, T);

  // shared memory: keys [T * G rows][DI] (swizzled), row bases [T, rounded up to even], q [G][Hi * W4 + 4],
  // w [G * Hi]
  uint8_t* keys = reinterpret_cast<uint8_t*>(smem_i32);
  long long* rbase = reinterpret_cast<long long*>(keys + (size_t)T * G * DI);
  const int gstride = Hi * W4 + 4;  // words; the 16-byte pad puts each g's block on its own banks
  int32_t* sq = reinterpret_cast<int32_t*>(rbase + ((T + 1) & ~1));  // 16-byte aligned
  int32_t* sw = sq + G * gstride;

  const int tid = threadIdx.x;
  if (tid < nt) {
    const int t = t0 + tid;
    const int page = block_table[(size_t)b * max_pages + t / page_size];
    long long base = -1;
    if (page >= 0 && page < num_pages)
      base = ((long long)page * page_size + t % page_size) * G * DI;
    else
      raise_error(SD_DEVERR_PAGE);
    rbase[tid] = base;
  }
  const int32_t* qw = reinterpret_cast<const int32_t*>(qi + (size_t)b * G * Hi * DI);
  {
    const int per_g = Hi * W4;
    int g = tid / per_g, r = tid % per_g;
    const int dg = kIdxThreads / per_g, dr = kIdxThreads % per_g;
    for (int i = tid; i < G * per_g; i += kIdxThreads) {
      sq[g * gstride + r] = qw[i];
      g += dg;
      r += dr;
      if (r >= per_g) {
        r -= per_g;
        ++g;
      }
    }
  }
  for (int i = tid; i < G * Hi; i += kIdxThreads) sw[i] = w[(size_t)b * G * Hi + i];
  __syncthreads();

  // stage the tile: piece i = token i / ppt, byte (i % ppt) * 16 of its G * DI row
  {
    const int ppt = G * kCpr;
    int tok = tid / ppt, off = (tid % ppt) * 16;
    const int dtok = kIdxThreads / ppt, doff = (kIdxThreads % ppt) * 16;
    for (int i = tid; i < nt * ppt; i += kIdxThreads) {
      const long long base = rbase[tok];
      const int row = i / kCpr, c = i % kCpr;  // row = tok * G + off / DI
      cp_async_16(keys + (size_t)row * DI + idx_swz<DI>(c, row) * 16, ki_pages + (base >= 0 ? base + off : 0),
                  base >= 0 ? 16 : 0);
      tok += dtok;
      off += doff;
      if (off >= ppt * 16) {
        off -= ppt * 16;
        ++tok;
      }
    }
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  // score the pairs: pair p = token p / G, KV head p % G, key row p
  int tok = tid / G, g = tid % G;
  const int dtok = kIdxThreads / G, dg = kIdxThreads % G;
  for (int p = tid; p < nt * G; p += kIdxThreads) {
    int32_t* dst = scores + ((size_t)b * G + g) * max_seqlen + t0 + tok;
    if (rbase[tok] < 0) {
      *dst = INT32_MIN;
    } else {
      int32_t kv[W4];
#pragma unroll
      for (int c = 0; c < kCpr; ++c) {
        const int4 v = *reinterpret_cast<const int4*>(keys + (size_t)p * DI + idx_swz<DI>(c, p) * 16);
        kv[4 * c + 0] = v.x;
        kv[4 * c + 1] = v.y;
        kv[4 * c + 2] = v.z;
        kv[4 * c + 3] = v.w;
      }
      const int32_t* qg = sq + g * gstride;
      int32_t acc = 0;
      for (int h = 0; h < Hi; ++h) {
        int32_t dot = 0;
#pragma unroll
        for (int c = 0; c < kCpr; ++c) {
          const int4 q4 = *reinterpret_cast<const int4*>(qg + h * W4 + 4 * c);
          dot = __dp4a(q4.x, kv[4 * c + 0], dot);
          dot = __dp4a(q4.y, kv[4 * c + 1], dot);
          dot = __dp4a(q4.z, kv[4 * c + 2], dot);
          dot = __dp4a(q4.w, kv[4 * c + 3], dot);
        }
        acc += sw[g * Hi + h] * max(dot, 0);
      }
      *dst = acc;
    }
    tok += dtok;
    g += dg;
    if (g >= G) {
      g -= G;
      ++tok;
    }
  }
}

inline size_t indexer_dp4a_smem(int G, int Hi, int Di) {
  const int T = indexer_dp4a_tokens(G, Di);
  return (size_t)T * G * Di + sizeof(long long) * ((T + 1) & ~1) +
         sizeof(int32_t) * ((size_t)G * (Hi * (Di / 4) + 4) + G * Hi);
}

}  // namespace sd
