// Indexer scores on the 5th-generation tensor cores (tcgen05, kind::i8):
//
//   s[b,g,t] = sum_h w[b,g,h] * max(0, sum_d qi[b,g,h,d] * ki[t,g,d])
//
// Per 128-token tile, the keys of the tile are the M = 128 operand A (K-major:
// a token's G * Di bytes, exactly the NHD page layout, stored as 128-byte
// column chunks of [128 tokens x 128 B]), the request's queries are operand B
// (N = G * HPG heads, K = G * Di), and the int32 products D[token, head] land
// in tensor memory, one TMEM lane per token. With one KV head (the MLA
// indexer, G = 1, Di = 128) B is the request's [HPG x 128] query block, loaded
// by TMA. With several KV heads (per-head selection) B is block-diagonal:
// head (g, h) holds qi[b,g,h] in the K columns of KV head g and zeros
// elsewhere, so one MMA chain scores every KV head's keys at once (the zeros
// cost tensor time that stays far below the key stream); the producer warp
// builds it in shared memory. The ReLU and the weighted head sums are then a
// per-thread loop over that thread's TMEM row, and each warp writes 32
// consecutive scores per KV head.
//
// Keys stream straight from the paged pool: the TMA engine copies each page
// of the tile (P rows x 128 B, 128-byte swizzle) into a shared-memory stage,
// addressed through the block table ("direct paged-pool scoring ... no Torch
// gather", "Add TriAttention KV-cache compression method", Key Design
// Decisions). Work is balanced over a persistent grid of one CTA per SM:
// the tiles of all requests form one list, and each CTA takes a contiguous
// share of it (requests of any length, no host-side schedule).
//
// Roles (320 threads): warp 0 issues TMA, warp 1 owns tensor memory and issues
// the MMAs, warps 2-9 run the epilogue as two sets of four (set e takes the
// tiles i = e mod 2; warp w reads TMEM lanes 32*(w%4)..+31). Stages are
// recycled through mbarriers; tile i accumulates into one of kUmmaAccs
// tensor-memory accumulators (i mod kUmmaAccs), so the MMAs run up to
// kUmmaAccs - 1 tiles ahead of the epilogue.
#pragma once

#include "sm100.cuh"

namespace sd {

constexpr int kUmmaTile = 128;     // tokens per tile (MMA M)
constexpr int kUmmaChunk = 128;    // bytes of a K-major column chunk (the 128-byte swizzle)
constexpr int kUmmaAccs = 4;       // accumulators in tensor memory (tile i uses i % 4)
constexpr int kUmmaEpiSets = 2;   // epilogue warp sets; set e reads the tiles i = e (mod 2)
constexpr int kUmmaThreads = 64 + 128 * kUmmaEpiSets;

// G KV heads of Di-byte keys, HPG indexer heads per KV head; TPS tiles of one
// request share a shared-memory stage, STAGES stages.
template <int G, int HPG, int DI, int TPS, int STAGES>
struct IndexerUmmaCfg {
  static constexpr int kHeads = G * HPG;            // MMA N (accumulator columns)
  static constexpr int kRowBytes = G * DI;          // key bytes per token (MMA K)
  static constexpr int kChunks = kRowBytes / kUmmaChunk;
  static constexpr int kTilesPerStage = TPS;
  static constexpr int kStages = STAGES;
  static constexpr int kChunkBytes = kUmmaTile * kUmmaChunk;  // 16 KB
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kStageBytes = TPS * kTileBytes;
  static constexpr int kQBytes = kChunks * kHeads * kUmmaChunk;
  static constexpr int kAccCols = kUmmaAccs * kHeads;
  static constexpr int kTmemCols = kAccCols <= 32 ? 32 : (kAccCols <= 64 ? 64 : (kAccCols <= 128 ? 128 : (kAccCols <= 256 ? 256 : 512)));
  static constexpr int kOffQ = STAGES * kStageBytes;
  static constexpr int kOffBar = kOffQ + 2 * kQBytes;
  static constexpr int kNumBars = 2 * STAGES + 2 + 2 + 2 * kUmmaAccs;
  static constexpr int kOffMisc = kOffBar + 8 * kNumBars;
  static constexpr int kBytes = kOffMisc + 16;
  static constexpr size_t kSmemAlloc = kBytes + 1024;  // slack to align the base to 1024 B
  static_assert(kRowBytes % kUmmaChunk == 0 && kHeads % 16 == 0 && kHeads <= 256, "MMA shape");
  static_assert(kAccCols <= 512 && kSmemAlloc <= 232448, "resources");
};
// The MLA indexer (one KV head, 64 heads of 128 bytes) and the per-head
// indexer (8 KV heads of 64 bytes, 4 heads each).
using IdxCfgMla = IndexerUmmaCfg<1, 64, 128, 4, 3>;
using IdxCfgPerHead = IndexerUmmaCfg<8, 4, 64, 1, 3>;

// Walks a contiguous range of the global tile list (request-major).

struct TileCursor {
  int b, tile, tiles_b, L;
  long long remaining;
  __device__ void init(const int32_t* seqlens, int B, int cap, long long first, long long count) {
    remaining = count;
    b = 0;
    tile = 0;
    long long skip = first;
    for (; b < B; ++b) {
      L = checked_seqlen(seqlens, b, cap);
      tiles_b = ceil_div(L, kUmmaTile);
      if (skip < tiles_b) break;
      skip -= tiles_b;
    }
    tile = static_cast<int>(skip);
  }
  __device__ bool valid() const { return remaining > 0; }
  __device__ void next(const int32_t* seqlens, int B, int cap) {
    --remaining;
    if (remaining <= 0) return;
    if (++tile < tiles_b) return;
    tile = 0;
    do {
      ++b;
      L = checked_seqlen(seqlens, b, cap);
      tiles_b = ceil_div(L, kUmmaTile);
    } while (tiles_b == 0 && b < B - 1);
  }
};

// A stage takes the cursor's tile and the following ones of the same
// request within the range, up to tiles_per_stage and to 32 pages (one
// block-table window); every tile but the stage's last is then a full 128
// tokens.
__device__ __forceinline__ int stage_tiles(const TileCursor& c, int pages_per_tile, int tiles_per_stage) {
  const long long left = c.remaining < (long long)(c.tiles_b - c.tile) ? c.remaining : (long long)(c.tiles_b - c.tile);
  const int cap = min(tiles_per_stage, 32 / pages_per_tile);
  return left < cap ? static_cast<int>(left) : cap;
}

__device__ __forceinline__ long long total_tiles(const int32_t* seqlens, int B, int cap) {
  long long n = 0;
  for (int b = 0; b < B; ++b) {
    int L = seqlens[b];
    L = L < 0 ? 0 : (L > cap ? cap : L);
    n += ceil_div(L, kUmmaTile);
  }
  return n;
}

// max(0, x) for an int32 dot product |x| < 2^31 - 2^23, on the FP32 pipe
// (twice the INT32 pipe's rate, which the weighted sum keeps busy): as a
// float, a nonnegative x is a nonnegative number (subnormals kept: no .ftz),
// a negative x a negative number or a NaN, and max.f32 returns +0 for both.
// Here |x| <= 128 * 128 * 128 = 2^21.
__device__ __forceinline__ int32_t relu_on_fp_pipe(uint32_t x) {
  uint32_t y;
  asm("max.f32 %0, %1, %2;" : "=r"(y) : "r"(x), "r"(0u));
  return static_cast<int32_t>(y);
}

template <class Cfg, int G, int HPG, int DI>
__global__ void __launch_bounds__(kUmmaThreads, 1) indexer_umma_kernel(
    const __grid_constant__ CUtensorMap tm_keys, const __grid_constant__ CUtensorMap tm_q,
    const int8_t* __restrict__ qi, const int32_t* __restrict__ w, const int32_t* __restrict__ block_table,
    const int32_t* __restrict__ seqlens, int32_t* __restrict__ scores, int B, int num_pages, int page_size,
    int max_pages, int max_seqlen) {
  using Lay = Cfg;
  constexpr int HI = Lay::kHeads;
  constexpr int kUmmaStages = Lay::kStages;
  extern __shared__ uint8_t smem_dyn[];
  const uint32_t raw = smem_u32(smem_dyn);
  uint8_t* smem = smem_dyn + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* kstage = smem;
  uint8_t* qbuf = smem + Lay::kOffQ;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + kUmmaStages;
  uint64_t* qfull = bars + 2 * kUmmaStages;
  uint64_t* qempty = qfull + 2;
  uint64_t* accfull = qempty + 2;
  uint64_t* accempty = accfull + kUmmaAccs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cap = min(max_seqlen, max_pages * page_size);
  const int pshift = __ffs(page_size) - 1;  // page sizes on this path are powers of two

  if (threadIdx.x == 0) {
    for (int i = 0; i < kUmmaStages; ++i) {
      sm100::mbar_init(&full[i], 1);
      sm100::mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      sm100::mbar_init(&qfull[i], 1);
      sm100::mbar_init(&qempty[i], 1);
    }
    for (int i = 0; i < kUmmaAccs; ++i) {
      sm100::mbar_init(&accfull[i], 1);
      sm100::mbar_init(&accempty[i], 128);
    }
    *abort_flag = 0;
    sm100::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    sm100::prefetch_tensormap(&tm_keys);
    sm100::prefetch_tensormap(&tm_q);
  }
  if (warp == 1) {
    sm100::tmem_alloc(tmem_slot, Lay::kTmemCols);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  // the set-up above reads no input: the previous kernel may still be running
  pdl_wait();
  pdl_trigger();
  const uint32_t tmem_base = *tmem_slot;

  const long long total = total_tiles(seqlens, B, cap);
  const long long first = total * blockIdx.x / gridDim.x;
  const long long count = total * (blockIdx.x + 1) / gridDim.x - first;
  if (threadIdx.x == 0) SD_PROBE_MARK(1, 0, count);

  if (warp == 0) {
    // ---------------- TMA producer (whole warp) ----------------
    // The 32 lanes keep a window of 32 consecutive block-table entries of the
    // current request (and the next window, loaded ahead), fetched in one
    // coalesced load, so the page lookups of 16+ tiles cost one memory round
    // trip. Windows start at tile boundaries, so the pages of a tile are
    // consecutive lanes: each such lane copies its own page. A page outside
    // the pool is copied from past the end of the tensor (zero fill), which
    // keeps the byte count of every stage fixed; the epilogue marks its
    // tokens invalid.
    TileCursor c;
    c.init(seqlens, B, cap, first, count);
    int stage = 0;
    uint32_t phase = 0;
    int nq = 0, cur_b = -1;
    const uint32_t page_bytes = static_cast<uint32_t>(page_size) * Lay::kRowBytes;
    const int ppt_shift = 7 - pshift;  // log2 of the pages of a tile
    // the keys are read once: keep them from evicting the scores, which the
    // top-k rereads right after this kernel
    const uint64_t evict_first = sm100::l2_policy_evict_first();
    const int oob_row = num_pages * page_size;
    int win_b = -1, win_p0 = 0, win_val = -1;
    int nxt_p0 = -1, nxt_val = -1;  // the following window of the same request, loaded ahead
    while (c.valid()) {
      if (c.b != cur_b) {
        const int slot = nq & 1;
        bool ok = true;
        if (lane == 0) ok = sm100::mbar_wait(&qempty[slot], ((nq >> 1) & 1) ^ 1) && !*abort_flag;
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          if (lane == 0) *abort_flag = 1;
          break;
        }
        if constexpr (G == 1) {
          // the request's [HI x 128] query block, by TMA
          if (lane == 0) {
            sm100::mbar_arrive_expect_tx(&qfull[slot], Lay::kQBytes);
            sm100::tma_load_2d(qbuf + slot * Lay::kQBytes, &tm_q, &qfull[slot], 0, c.b * HI);
          }
        } else {
          // the block-diagonal query operand: 16-byte granule j of row n in
          // chunk cc covers K bytes 128 cc + 16 j, which belong to KV head
          // (128 cc + 16 j) / DI; row n = g * HPG + h is qi[b,g,h] there and
          // zero elsewhere (rows in the 128-byte swizzle)
          uint8_t* qs = qbuf + slot * Lay::kQBytes;
          for (int idx = lane; idx < Lay::kChunks * HI * 8; idx += 32) {
            const int cc = idx / (HI * 8), n = (idx / 8) % HI, j = idx % 8;
            const int kb = kUmmaChunk * cc + 16 * j;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (kb / DI == n / HPG)
              v = __ldg(reinterpret_cast<const uint4*>(qi + ((size_t)c.b * HI + n) * DI + (kb % DI)));
            *reinterpret_cast<uint4*>(qs + cc * HI * kUmmaChunk + n * kUmmaChunk + ((j ^ (n & 7)) << 4)) = v;
          }
          sm100::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) sm100::mbar_arrive(&qfull[slot]);
        }
        cur_b = c.b;
        ++nq;
      }
      const int t0 = c.tile * kUmmaTile;
      const int p_first = t0 >> pshift;
      const int nt = stage_tiles(c, kUmmaTile >> pshift, Lay::kTilesPerStage);
      const int npages = (min(kUmmaTile * nt, c.L - t0) + page_size - 1) >> pshift;
      if (c.b != win_b || p_first + npages > win_p0 + 32) {
        if (c.b == win_b && p_first == nxt_p0) {
          win_val = nxt_val;  // loaded one window ago: no round trip on this path
        } else {
          const int p = p_first + lane;
          win_val = p < max_pages ? block_table[(size_t)c.b * max_pages + p] : -1;
        }
        win_b = c.b;
        win_p0 = p_first;
        nxt_p0 = win_p0 + 32;
        const int pn = nxt_p0 + lane;
        nxt_val = pn < max_pages ? block_table[(size_t)c.b * max_pages + pn] : -1;
      }
      const int off = lane - (p_first - win_p0);  // this lane's page within the tile
      bool ok = true;
      if (lane == 0) {
        ok = sm100::mbar_wait(&empty[stage], phase ^ 1) && (stage != 0 || !*abort_flag);
        if (ok) sm100::mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(npages) * page_bytes);
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      if (off >= 0 && off < npages) {
        // page `off` of the stage: tile off / ppt, rows (off % ppt) * P of
        // each of its column chunks
        const int row = (win_val >= 0 && win_val < num_pages) ? win_val * page_size : oob_row;
        uint8_t* dst = kstage + stage * Lay::kStageBytes + (off >> ppt_shift) * Lay::kTileBytes +
                       (off & ((1 << ppt_shift) - 1)) * page_size * kUmmaChunk;
#pragma unroll
        for (int cc = 0; cc < Lay::kChunks; ++cc)
          sm100::tma_load_2d_hint(dst + cc * Lay::kChunkBytes, &tm_keys, &full[stage], cc * kUmmaChunk, row,
                                  evict_first);
      }
      if (++stage == kUmmaStages) { stage = 0; phase ^= 1; }
      for (int j = 0; j < nt; ++j) c.next(seqlens, B, cap);
    }
    if (lane == 0) SD_PROBE_MARK(1, 1, 0);
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (sm100::elect_one()) {
      constexpr uint32_t idesc = sm100::idesc_i8(kUmmaTile, HI);
      TileCursor c;
      c.init(seqlens, B, cap, first, count);
      int stage = 0, acc = 0;
      uint32_t phase = 0, accphase = 0;
      int nq = 0, cur_b = -1;
      while (c.valid() && !*abort_flag) {
        if (c.b != cur_b) {
          if (!sm100::mbar_wait(&qfull[nq & 1], (nq >> 1) & 1)) { *abort_flag = 1; break; }
          cur_b = c.b;
          ++nq;
        }
        const int slot = (nq - 1) & 1;
        const int ntiles = stage_tiles(c, kUmmaTile >> pshift, Lay::kTilesPerStage);
        if (!sm100::mbar_wait(&full[stage], phase)) { *abort_flag = 1; break; }
        if (blockIdx.x % 37 == 0) SD_PROBE_MARK(1, 10, stage + kUmmaStages * static_cast<int>(phase));
        const uint32_t b0 = smem_u32(qbuf + slot * Lay::kQBytes);
        bool ok = true;
        for (int j = 0; j < ntiles; ++j) {
          if (!sm100::mbar_wait(&accempty[acc], accphase ^ 1)) { ok = false; break; }
          sm100::tc_fence_after();
          const uint32_t a0 = smem_u32(kstage + stage * Lay::kStageBytes + j * Lay::kTileBytes);
          const uint32_t d = tmem_base + acc * HI;
#pragma unroll
          for (int cc = 0; cc < Lay::kChunks; ++cc)
#pragma unroll
            for (int k = 0; k < kUmmaChunk / 32; ++k)
              sm100::mma_i8_ss(d, sm100::smem_desc_k_sw128(a0 + cc * Lay::kChunkBytes + 32 * k),
                               sm100::smem_desc_k_sw128(b0 + cc * HI * kUmmaChunk + 32 * k), idesc, (cc | k) > 0);
          sm100::mma_commit(&accfull[acc]);
          if (++acc == kUmmaAccs) { acc = 0; accphase ^= 1; }
        }
        if (!ok) { *abort_flag = 1; break; }
        sm100::mma_commit(&empty[stage]);
        const int this_b = c.b;
        for (int j = 0; j < ntiles; ++j) c.next(seqlens, B, cap);
        if (!c.valid() || c.b != this_b) sm100::mma_commit(&qempty[slot]);
        if (++stage == kUmmaStages) { stage = 0; phase ^= 1; }
      }
      SD_PROBE_MARK(1, 2, 0);
    }
  } else {
    // ---------------- epilogue: ReLU, weighted head sum, store ----------------
    // Two sets of four warps take alternate tiles (set e: tiles i = e mod 2,
    // accumulator e), so each set has two tile periods per tile. A warp reads
    // its TMEM quadrant (warp % 4); the accumulator is released as soon as
    // its row is in registers; the block-table entry that validates this
    // thread's token is loaded one tile of the set ahead.
    static_assert(kUmmaAccs % kUmmaEpiSets == 0, "each set cycles through its own accumulators");
    const int set = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    int ti = set;  // this CTA's tile number: accumulator ti % kUmmaAccs
    TileCursor c;
    c.init(seqlens, B, cap, first, count);
    for (int i = 0; i < set; ++i) c.next(seqlens, B, cap);
    int cur_b = -1;
    int32_t wreg[HI];
    auto page_of = [&](const TileCursor& cc) -> int {
      const int t = cc.tile * kUmmaTile + row;
      return (cc.valid() && t < cc.L) ? block_table[(size_t)cc.b * max_pages + (t >> pshift)] : 0;
    };
    int phys_next = page_of(c);
    while (c.valid() && !*abort_flag) {
      if (c.b != cur_b) {
#pragma unroll
        for (int h = 0; h < HI; ++h) wreg[h] = __ldg(w + (size_t)c.b * HI + h);
        cur_b = c.b;
      }
      const int t = c.tile * kUmmaTile + row;
      const int phys = phys_next;
      TileCursor cn = c;
      for (int i = 0; i < kUmmaEpiSets; ++i) cn.next(seqlens, B, cap);
      phys_next = page_of(cn);
      const int acc = ti % kUmmaAccs;
      const bool ok = sm100::mbar_wait(&accfull[acc], static_cast<uint32_t>((ti / kUmmaAccs) & 1));
      __syncwarp();  // tcgen05.ld is warp-collective: reconverge after the polling loop
      if (!ok) { *abort_flag = 1; break; }
      if (blockIdx.x % 37 == 0 && quarter == 0 && lane == 0) SD_PROBE_MARK(1, 11 + set, ti >> 1);
      sm100::tc_fence_after();
      uint32_t r[HI];
#pragma unroll
      for (int j = 0; j < HI / 32; ++j)
        sm100::tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * HI + j * 32,
                                  *reinterpret_cast<uint32_t(*)[32]>(r + 32 * j));
      sm100::tmem_ld_wait();
      sm100::tc_fence_before();
      sm100::mbar_arrive(&accempty[acc]);
      if (t < c.L) {
        const bool bad = phys < 0 || phys >= num_pages;
        if (bad) raise_error(SD_DEVERR_PAGE);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          // independent partial sums (a single chain would serialize the IMADs)
          constexpr int kPart = HPG >= 8 ? 8 : HPG;
          int32_t part[kPart];
#pragma unroll
          for (int i = 0; i < kPart; ++i) part[i] = 0;
#pragma unroll
          for (int i = 0; i < HPG; ++i)
            part[i % kPart] += wreg[g * HPG + i] * relu_on_fp_pipe(r[g * HPG + i]);
          int32_t s = 0;
#pragma unroll
          for (int i = 0; i < kPart; ++i) s += part[i];
          scores[((size_t)c.b * G + g) * max_seqlen + t] = bad ? INT32_MIN : s;
        }
      }
      ti += kUmmaEpiSets;
      c = cn;
    }
    if (quarter == 0 && lane == 0) SD_PROBE_MARK(1, 3 + set, 0);
  }

  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    sm100::tmem_dealloc(tmem_base, Lay::kTmemCols);
  }
}

}  // namespace sd
