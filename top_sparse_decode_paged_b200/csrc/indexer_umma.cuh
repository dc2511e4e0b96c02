// Indexer scores on the 5th-generation tensor cores (tcgen05, kind::i8) for a
// single KV head with 128-byte key rows (Di = 128) and HI indexer heads:
//
//   s[b,t] = sum_h w[b,h] * max(0, sum_d qi[b,h,d] * ki[t,d])
//
// Per 128-token tile, the keys of the tile are the M = 128 operand A (K-major,
// one 128-byte row per token, exactly the NHD page layout), the request's
// queries are operand B (N = HI heads, K-major), and the int32 products
// D[token, head] land in tensor memory, one TMEM lane per token. The ReLU and
// the weighted head sum are then a per-thread loop over that thread's TMEM
// row, and each warp writes 32 consecutive scores.
//
// Keys stream straight from the paged pool: the TMA engine copies each page
// of the tile (P rows x 128 B, 128-byte swizzle) into a shared-memory stage,
// addressed through the block table ("direct paged-pool scoring ... no Torch
// gather", "Add TriAttention KV-cache compression method", Key Design
// Decisions). Work is balanced over a persistent grid of one CTA per SM:
// the tiles of all requests form one list, and each CTA takes a contiguous
// share of it (requests of any length, no host-side schedule).
//
// Roles (192 threads): warp 0 issues TMA, warp 1 owns tensor memory and issues
// the MMAs, warps 2-5 run the epilogue (warp w reads TMEM lanes 32*(w%4)..+31).
// Stages are recycled through mbarriers; accumulators are double-buffered.
#pragma once

#include "sm100.cuh"

namespace sd {

constexpr int kUmmaTile = 128;     // tokens per tile (MMA M)
constexpr int kUmmaRowBytes = 128; // Di = 128 int8
constexpr int kUmmaStages = 6;
constexpr int kUmmaTilesPerStage = 2;  // consecutive tiles of one request share a stage
constexpr int kUmmaAccs = 2;       // accumulators in tensor memory (tile i uses i % 2)
constexpr int kUmmaEpiSets = 2;   // epilogue warp sets; set e reads the tiles i = e (mod 2)
constexpr int kUmmaThreads = 64 + 128 * kUmmaEpiSets;

template <int HI>
struct IndexerUmmaLayout {
  static constexpr int kTileBytes = kUmmaTile * kUmmaRowBytes;  // 16 KB
  static constexpr int kStageBytes = kUmmaTilesPerStage * kTileBytes;
  static constexpr int kQBytes = HI * kUmmaRowBytes;
  static constexpr int kAccCols = kUmmaAccs * HI;
  static constexpr int kTmemCols = kAccCols <= 32 ? 32 : (kAccCols <= 64 ? 64 : (kAccCols <= 128 ? 128 : (kAccCols <= 256 ? 256 : 512)));
  static constexpr int kOffQ = kUmmaStages * kStageBytes;
  static constexpr int kOffBar = kOffQ + 2 * kQBytes;
  static constexpr int kNumBars = 2 * kUmmaStages + 2 + 2 + 2 * kUmmaAccs;
  static constexpr int kOffMisc = kOffBar + 8 * kNumBars;
  static constexpr int kBytes = kOffMisc + 16;
  static constexpr size_t kSmemAlloc = kBytes + 1024;  // slack to align the base to 1024 B
};

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
// request within the range, up to kUmmaTilesPerStage and to 32 pages (one
// block-table window); every tile but the stage's last is then a full 128
// tokens.
__device__ __forceinline__ int stage_tiles(const TileCursor& c, int pages_per_tile) {
  const long long left = c.remaining < (long long)(c.tiles_b - c.tile) ? c.remaining : (long long)(c.tiles_b - c.tile);
  const int cap = min(kUmmaTilesPerStage, 32 / pages_per_tile);
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

template <int HI>
__global__ void __launch_bounds__(kUmmaThreads, 1) indexer_umma_kernel(
    const __grid_constant__ CUtensorMap tm_keys, const __grid_constant__ CUtensorMap tm_q,
    const int32_t* __restrict__ w, const int32_t* __restrict__ block_table,
    const int32_t* __restrict__ seqlens, int32_t* __restrict__ scores, int B, int num_pages, int page_size,
    int max_pages, int max_seqlen) {
  using Lay = IndexerUmmaLayout<HI>;
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
    const uint32_t page_bytes = static_cast<uint32_t>(page_size) * kUmmaRowBytes;
    const int oob_row = num_pages * page_size;
    int win_b = -1, win_p0 = 0, win_val = -1;
    int nxt_p0 = -1, nxt_val = -1;  // the following window of the same request, loaded ahead
    while (c.valid()) {
      if (c.b != cur_b) {
        const int slot = nq & 1;
        bool ok = true;
        if (lane == 0) {
          ok = sm100::mbar_wait(&qempty[slot], ((nq >> 1) & 1) ^ 1) && !*abort_flag;
          if (ok) {
            sm100::mbar_arrive_expect_tx(&qfull[slot], Lay::kQBytes);
            sm100::tma_load_2d(qbuf + slot * Lay::kQBytes, &tm_q, &qfull[slot], 0, c.b * HI);
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          if (lane == 0) *abort_flag = 1;
          break;
        }
        cur_b = c.b;
        ++nq;
      }
      const int t0 = c.tile * kUmmaTile;
      const int p_first = t0 >> pshift;
      const int nt = stage_tiles(c, kUmmaTile >> pshift);
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
        const int row = (win_val >= 0 && win_val < num_pages) ? win_val * page_size : oob_row;
        sm100::tma_load_2d(kstage + stage * Lay::kStageBytes + off * page_bytes, &tm_keys, &full[stage], 0, row);
      }
      if (++stage == kUmmaStages) { stage = 0; phase ^= 1; }
      for (int j = 0; j < nt; ++j) c.next(seqlens, B, cap);
    }
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
        const int ntiles = stage_tiles(c, kUmmaTile >> pshift);
        if (!sm100::mbar_wait(&full[stage], phase)) { *abort_flag = 1; break; }
        const uint32_t b0 = smem_u32(qbuf + slot * Lay::kQBytes);
        bool ok = true;
        for (int j = 0; j < ntiles; ++j) {
          if (!sm100::mbar_wait(&accempty[acc], accphase ^ 1)) { ok = false; break; }
          sm100::tc_fence_after();
          const uint32_t a0 = smem_u32(kstage + stage * Lay::kStageBytes + j * Lay::kTileBytes);
          const uint32_t d = tmem_base + acc * HI;
#pragma unroll
          for (int k = 0; k < kUmmaRowBytes / 32; ++k)
            sm100::mma_i8_ss(d, sm100::smem_desc_k_sw128(a0 + 32 * k), sm100::smem_desc_k_sw128(b0 + 32 * k),
                             idesc, k > 0);
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
    }
  } else {
    // ---------------- epilogue: ReLU, weighted head sum, store ----------------
    // Two sets of four warps take alternate tiles (set e: tiles i = e mod 2,
    // accumulator e), so each set has two tile periods per tile. A warp reads
    // its TMEM quadrant (warp % 4); the accumulator is released as soon as
    // its row is in registers; the block-table entry that validates this
    // thread's token is loaded one tile of the set ahead.
    static_assert(kUmmaAccs == kUmmaEpiSets, "one accumulator per epilogue set");
    const int set = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int acc = set;
    uint32_t accphase = 0;
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
      const bool ok = sm100::mbar_wait(&accfull[acc], accphase);
      __syncwarp();  // tcgen05.ld is warp-collective: reconverge after the polling loop
      if (!ok) { *abort_flag = 1; break; }
      sm100::tc_fence_after();
      uint32_t r[HI];
#pragma unroll
      for (int j = 0; j < HI / 32; ++j)
        sm100::tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * HI + j * 32,
                                  *reinterpret_cast<uint32_t(*)[32]>(r + 32 * j));
      sm100::tmem_ld_wait();
      sm100::tc_fence_before();
      sm100::mbar_arrive(&accempty[acc]);
      // eight independent partial sums (a single chain would serialize 64 IMADs)
      int32_t part[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
      for (int i = 0; i < HI; ++i) part[i & 7] += wreg[i] * max(static_cast<int32_t>(r[i]), 0);
      const int32_t s0 = (part[0] + part[1]) + (part[2] + part[3]);
      const int32_t s1 = (part[4] + part[5]) + (part[6] + part[7]);
      int32_t s = s0 + s1;
      if (t < c.L) {
        if (phys < 0 || phys >= num_pages) {
          raise_error(SD_DEVERR_PAGE);
          s = INT32_MIN;
        }
        scores[(size_t)c.b * max_seqlen + t] = s;
      }
      accphase ^= 1;
      c = cn;
    }
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
