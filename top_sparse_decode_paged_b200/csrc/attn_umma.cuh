// Sparse MLA decode attention on the 5th-generation tensor cores (tcgen05),
// for 128 query heads sharing one 576-wide latent row per token (V = the
// first 512 columns): the selected-token MLA of "Add DSA Vanilla sparse
// attention" (Walkthrough), consuming the top-k buffer of the DSA decode
// step ("Overlap DSA heuristic prev_topk write-back on the aux stream").
//
// Tensor memory holds 128 lanes x 512 fp32 columns, and the full output of one
// request (128 heads x 512 values) alone would fill it. So each tile range is
// served by two CTAs, each owning half of the value columns:
//   TMEM cols [0,256)   O half  (128 heads x 256 values, fp32, accumulated)
//   TMEM cols [256,512) S       (128 heads x 256 selected tokens, fp32)
//   TMEM cols [256,384) P       (bf16 pairs, written over S by the softmax)
// Both CTAs compute the same S = Q K^T (M = 128 heads, N = 256 tokens,
// K = 576); each then runs O += P V over its half (A = P from tensor memory,
// B = V from shared memory).
//
// Data movement: a four-slot ring of 48 KB slots. For each of the nine S steps
// of a tile, a slot receives Q[:, 64 columns] (16 KB, one TMA tile; Q stays in
// L2) and the tile's K[:, same columns] (32 KB, 256 rows x 128 bytes, gathered
// by four copy warps with coalesced cp.async: 8 lanes per 128-byte row piece,
// destination swizzle applied per 16-byte lane, skipped selections copy zeros).
// The four V chunks of this CTA's half use the gather part of a slot. Keeping
// Q out of shared memory is what buys the ring depth. A TMA tile::gather4 gather measured well below this on the part: it
// moves one 128-byte row piece per ~20 cycles per SM. Each tile streams the nine K
// chunks for S, then the four V chunks of this CTA's half; the same chunk
// layout serves as the K-major B of S and as the MN-major B of P V. Whole rows
// of the next tile are prefetched into L2 while the current one is consumed.
//
// Softmax: the thread of TMEM lane h owns head h's row, so the row max and
// sum stay in registers. The running max is updated lazily: O is rescaled
// only when a tile's max exceeds the reference by more than 2^8, so most tiles
// skip the read-modify-write of O.
//
// Work: all requests' tiles (ceil(min(k, L) / 256) per request) form one list
// that is cut into equal contiguous ranges, one per CTA pair. A range that
// covers parts of several requests writes one partial (O, m, l) per request.
// The combine kernel merges them.
//
// Roles (288 threads): warps 0-3 copy, warps 4-7 run the softmax and write
// partials (warp w owns TMEM lanes 32*(w%4)..+31), warp 8 issues the MMAs. Every wait is bounded (a timeout flags SD_DEVERR_TIMEOUT).
#pragma once

#include "sm100.cuh"

namespace sd {

constexpr int kAuTile = 256;               // selected tokens per tile (N of S)
constexpr int kAuHeads = 128;              // M
constexpr int kAuDk = 576, kAuDv = 512;
constexpr int kAuQChunks = kAuDk / 64;     // 9
constexpr int kAuVChunks = kAuDv / 2 / 64; // 4 per value half
constexpr int kAuChunkBytes = kAuTile * 128;   // 32 KB: 256 rows x 64 columns
constexpr int kAuQChunkBytes = kAuHeads * 128; // 16 KB: 128 heads x 64 columns
constexpr int kAuSlotBytes = kAuQChunkBytes + kAuChunkBytes;  // one ring slot
constexpr int kAuSlots = 4;
constexpr int kAuThreads = 288;
constexpr int kAuRanges = 74;              // CTA pairs: 148 CTAs, one per SM
constexpr float kAuRescaleLog2 = 8.0f;     // lazy rescale threshold (log2 units)
constexpr int kAuPrefetchTiles = 3;       // L2 prefetch distance (tiles)
constexpr int kMaxTopK = 2048;            // largest k the library accepts

struct AttnUmmaLayout {
  static constexpr int kOffRing = 0;
  static constexpr int kOffBar = kAuSlots * kAuSlotBytes;           // 196608
  static constexpr int kNumBars = 2 * kAuSlots + 3;
  static constexpr int kOffMask = kOffBar + 8 * kNumBars;
  static constexpr int kOffMisc = kOffMask + 2 * 8 * 4;
  static constexpr int kBytes = kOffMisc + 16;
  static constexpr size_t kSmemAlloc = kBytes + 1024;
};

// Walks a contiguous range of the attention tile list (request-major).
struct AttnCursor {
  int b, tile, tiles_b, L;
  long long remaining;
  __device__ static int tiles_of(int L, int k) { return ceil_div(min(k, L), kAuTile); }
  __device__ void init(const int32_t* seqlens, int B, int cap, int k, long long first, long long count) {
    remaining = count;
    long long skip = first;
    for (b = 0; b < B; ++b) {
      L = checked_seqlen(seqlens, b, cap);
      tiles_b = tiles_of(L, k);
      if (skip < tiles_b) break;
      skip -= tiles_b;
    }
    tile = static_cast<int>(skip);
  }
  __device__ bool valid() const { return remaining > 0; }
  __device__ void next(const int32_t* seqlens, int B, int cap, int k) {
    if (--remaining <= 0) return;
    if (++tile < tiles_b) return;
    tile = 0;
    do {
      ++b;
      L = checked_seqlen(seqlens, b, cap);
      tiles_b = tiles_of(L, k);
    } while (tiles_b == 0 && b < B - 1);
  }
};

__device__ __forceinline__ long long attn_total_tiles(const int32_t* seqlens, int B, int cap, int k) {
  long long n = 0;
  for (int b = 0; b < B; ++b) {
    int L = seqlens[b];
    L = L < 0 ? 0 : (L > cap ? cap : L);
    n += ceil_div(min(k, L), kAuTile);
  }
  return n;
}

// Row id (page * P + slot) of selection slot `s` of request b, or -1.
__device__ __forceinline__ long long attn_row_of(const int32_t* indices, const int32_t* block_table, int b, int s,
                                                 int kb, int k, int L, int page_size, int max_pages, int num_pages) {
  if (s >= kb) return -1;
  const int t = indices[(size_t)b * k + s];
  if (t < 0) return -1;
  if (t >= L) {
    raise_error(SD_DEVERR_INDEX);
    return -1;
  }
  const int page = block_table[(size_t)b * max_pages + t / page_size];
  if (page < 0 || page >= num_pages) {
    raise_error(SD_DEVERR_PAGE);
    return -1;
  }
  return (long long)page * page_size + (t % page_size);
}

__global__ void __launch_bounds__(kAuThreads, 1) attn_mla_umma_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
    const __nv_bfloat16* __restrict__ kv,
    const int32_t* __restrict__ block_table, const int32_t* __restrict__ seqlens,
    const int32_t* __restrict__ indices, int B, int k, int num_pages, int page_size, int max_pages,
    int seqlen_cap, float scale_log2, float* __restrict__ part_o, float2* __restrict__ part_ml) {
  using Lay = AttnUmmaLayout;
  extern __shared__ uint8_t smem_dyn[];
  const uint32_t raw = smem_u32(smem_dyn);
  uint8_t* smem = smem_dyn + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* ring = smem + Lay::kOffRing;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kOffBar);
  uint64_t* chunk_full = bars;                   // [kAuSlots]: 128 copy arrivals + 1 TMA issuer
  uint64_t* chunk_empty = bars + kAuSlots;       // [kAuSlots]: MMA commit
  uint64_t* s_full = bars + 2 * kAuSlots;        // MMA commit
  uint64_t* p_full = bars + 2 * kAuSlots + 1;    // 128 softmax arrivals
  uint64_t* pv_done = bars + 2 * kAuSlots + 2;   // MMA commit
  uint32_t* mask_words = reinterpret_cast<uint32_t*>(smem + Lay::kOffMask);  // [2][8]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_ranges = gridDim.x / 2;
  const int range = blockIdx.x % n_ranges;
  const int half = blockIdx.x / n_ranges;  // which 256 value columns this CTA owns

  if (threadIdx.x == 0) {
    for (int i = 0; i < kAuSlots; ++i) {
      sm100::mbar_init(&chunk_full[i], 129);
      sm100::mbar_init(&chunk_empty[i], 1);
    }
    sm100::mbar_init(s_full, 1);
    sm100::mbar_init(p_full, 128);
    sm100::mbar_init(pv_done, 1);
    *abort_flag = 0;
    sm100::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    sm100::prefetch_tensormap(&tm_q);
    sm100::prefetch_tensormap(&tm_kv);
  }
  if (warp == 8) {
    sm100::tmem_alloc(tmem_slot, 512);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_o = tmem;          // cols [0,256)
  const uint32_t tm_s = tmem + 256;    // cols [256,512); P over [256,384)

  const long long total = attn_total_tiles(seqlens, B, seqlen_cap, k);
  const long long first = total * range / n_ranges;
  const long long count = total * (range + 1) / n_ranges - first;

  if (warp < 4) {
    // ------------------------------ copies ------------------------------
    // Each S chunk c of a tile fills one ring slot with Q[:, 64c..64c+63] (a
    // 16 KB TMA tile; Q is small and stays in L2) and the tile's K[:, 64c..]
    // (32 KB gathered with cp.async). A V chunk fills the gather part only.
    // The gather is coalesced: in each copy instruction 8 lanes fetch one
    // 128-byte row piece, so a warp moves 4 pieces (512 B); the 16-byte
    // swizzle of the destination is applied per lane. Thread pt fetches rows
    // 64*warp + 4*i + lane/8 (i = 0..15), 16-byte column j = lane % 8.
    const int pt = threadIdx.x;  // 0..127
    const int jseg = lane & 7;
    AttnCursor c;
    c.init(seqlens, B, seqlen_cap, k, first, count);
    long long n = 0;  // ring uses
    bool ok = true;
    while (c.valid() && ok) {
      const int kb = min(k, c.L);
      const int s0 = c.tile * kAuTile;
      int row[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const long long r = attn_row_of(indices, block_table, c.b, s0 + 64 * warp + 4 * i + (lane >> 3), kb, k, c.L,
                                        page_size, max_pages, num_pages);
        row[i] = static_cast<int>(r);  // -1: skipped, copied as zeros
      }
      // Whole selected rows into L2 ahead of their gathers: the tiles up to
      // kAuPrefetchTiles ahead (on the first tile, those in between too).
      {
        AttnCursor nx = c;
        for (int ahead = 0; ahead <= kAuPrefetchTiles && nx.valid(); ++ahead) {
          if (ahead == kAuPrefetchTiles || (n == 0 && ahead < kAuPrefetchTiles)) {
            const int nkb = min(k, nx.L);
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
              const long long r = attn_row_of(indices, block_table, nx.b, nx.tile * kAuTile + pt + 128 * rr, nkb, k,
                                              nx.L, page_size, max_pages, num_pages);
              if (r >= 0) sm100::prefetch_l2_bulk(kv + r * kAuDk, kAuDk * 2);
            }
          }
          nx.next(seqlens, B, seqlen_cap, k);
        }
      }
      for (int ci = 0; ci < kAuQChunks + kAuVChunks && ok; ++ci, ++n) {
        const bool is_s = ci < kAuQChunks;
        const int cc = is_s ? ci : half * kAuVChunks + (ci - kAuQChunks);
        const int slot = static_cast<int>(n % kAuSlots);
        ok = sm100::mbar_wait(&chunk_empty[slot], static_cast<uint32_t>((n / kAuSlots) & 1) ^ 1) && !*abort_flag;
        if (!ok) break;
        uint8_t* slot_base = ring + slot * kAuSlotBytes;
        if (pt == 0) {
          sm100::mbar_arrive_expect_tx(&chunk_full[slot], is_s ? kAuQChunkBytes : 0);
          if (is_s) sm100::tma_load_2d(slot_base, &tm_q, &chunk_full[slot], cc * 64, c.b * kAuHeads);
        }
        uint8_t* dst_base = slot_base + kAuQChunkBytes;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int r = 64 * warp + 4 * i + (lane >> 3);
          const int rw = row[i];
          const __nv_bfloat16* src = kv + (long long)(rw >= 0 ? rw : 0) * kAuDk + cc * 64 + jseg * 8;
          cp_async_16(dst_base + r * 128 + ((jseg ^ (r & 7)) << 4), src, rw >= 0 ? 16 : 0);
        }
        sm100::cp_async_arrive_noinc(&chunk_full[slot]);
      }
      c.next(seqlens, B, seqlen_cap, k);
    }
    cp_async_wait<0>();
    if (!ok) *abort_flag = 1;
  } else if (warp < 8) {
    // ------------------------ softmax and partials ------------------------
    const int st = threadIdx.x - 128;         // 0..127
    const int sw = warp - 4;                  // 0..3 (mask word owner)
    const int quarter = warp & 3;
    const int head = quarter * 32 + lane;     // TMEM lane == head
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    AttnCursor c;
    c.init(seqlens, B, seqlen_cap, k, first, count);
    int ntile = 0;
    bool seg_first = true;
    float m_ref = -INFINITY, l_sum = 0.f;
    while (c.valid()) {
      const int kb = min(k, c.L);
      const int s0 = c.tile * kAuTile;
      uint32_t* mw = mask_words + (ntile & 1) * 8;
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const bool v = attn_row_of(indices, block_table, c.b, s0 + st + rr * 128, kb, k, c.L, page_size,
                                   max_pages, num_pages) >= 0;
        const uint32_t bal = __ballot_sync(0xffffffffu, v);
        if (lane == 0) mw[rr * 4 + sw] = bal;
      }
      // wait for S, then one barrier both publishes the mask words and makes
      // the exit decision uniform over the 128 softmax threads
      bool ok = sm100::mbar_wait(s_full, ntile & 1) && !*abort_flag;
      ok = sm100::named_bar_and(1, 128, ok);
      if (!ok) { *abort_flag = 1; break; }
      uint32_t mask[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) mask[j] = mw[j];
      sm100::tc_fence_after();

      // pass 1: row max over the valid tokens
      float mx = -INFINITY;
#pragma unroll 1
      for (int j = 0; j < 8; ++j) {
        uint32_t r[32];
        sm100::tmem_ld_32x32b_x32(tm_s + lane_base + 32 * j, r);
        sm100::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if ((mask[j] >> i) & 1u) mx = fmaxf(mx, __uint_as_float(r[i]) * scale_log2);
      }
      const float m_tile = mx;  // max of the scaled logits (any sign of scale)
      const bool need = m_tile > m_ref + kAuRescaleLog2 || (m_ref == -INFINITY && m_tile > -INFINITY);
      float alpha = 1.f;
      if (need) {
        alpha = exp2f(m_ref - m_tile);  // 0 when m_ref is -inf
        l_sum *= alpha;
        m_ref = m_tile;
      }
      // O holds earlier tiles of this segment: scale rows whose reference moved
      // (warp-uniform branch: tcgen05.ld/st are warp-collective)
      if (__any_sync(0xffffffffu, need) && !seg_first) {
#pragma unroll 1
        for (int j = 0; j < 8; ++j) {
          uint32_t r[32];
          sm100::tmem_ld_32x32b_x32(tm_o + lane_base + 32 * j, r);
          sm100::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          sm100::tmem_st_32x32b_x32(tm_o + lane_base + 32 * j, r);
        }
        sm100::tmem_st_wait();
      }
      const float m_use = m_ref == -INFINITY ? 0.f : m_ref;

      // pass 2: P = 2^(s * scale_log2 - m_ref) as bf16, written over S
#pragma unroll 1
      for (int j = 0; j < 8; ++j) {
        uint32_t r[32], pk[16];
        sm100::tmem_ld_32x32b_x32(tm_s + lane_base + 32 * j, r);
        sm100::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = ((mask[j] >> (2 * i)) & 1u) ? sm100::ex2_approx(__uint_as_float(r[2 * i]) * scale_log2 - m_use) : 0.f;
          const float p1 =
              ((mask[j] >> (2 * i + 1)) & 1u) ? sm100::ex2_approx(__uint_as_float(r[2 * i + 1]) * scale_log2 - m_use) : 0.f;
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
          l_sum += __low2float(h2) + __high2float(h2);
          pk[i] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        sm100::tmem_st_32x32b_x16(tm_s + lane_base + 16 * j, pk);
      }
      sm100::tmem_st_wait();
      sm100::tc_fence_before();
      sm100::mbar_arrive(p_full);

      const int this_b = c.b;
      c.next(seqlens, B, seqlen_cap, k);
      const bool seg_end = !c.valid() || c.b != this_b;
      if (seg_end) {
        bool okd = sm100::mbar_wait(pv_done, ntile & 1) && !*abort_flag;
        okd = sm100::named_bar_and(2, 128, okd);
        if (!okd) { *abort_flag = 1; break; }
        sm100::tc_fence_after();
        const size_t slot = static_cast<size_t>(range) + this_b;
        float* dst = part_o + ((slot * 2 + half) * kAuHeads + head) * (kAuDv / 2);
#pragma unroll 1
        for (int j = 0; j < 8; ++j) {
          uint32_t r[32];
          sm100::tmem_ld_32x32b_x32(tm_o + lane_base + 32 * j, r);
          sm100::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + 32 * j + i) =
                make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]), __uint_as_float(r[i + 2]),
                            __uint_as_float(r[i + 3]));
        }
        if (half == 0) part_ml[slot * kAuHeads + head] = make_float2(m_ref, l_sum);
        sm100::tc_fence_before();
        m_ref = -INFINITY;
        l_sum = 0.f;
      }
      seg_first = seg_end;
      ++ntile;
    }
  } else {
    // ------------------------------ MMA issue ------------------------------
    if (sm100::elect_one()) {
      constexpr uint32_t idesc_s = sm100::idesc_bf16(kAuHeads, kAuTile, false, false);
      constexpr uint32_t idesc_pv = sm100::idesc_bf16(kAuHeads, 64, false, true);
      AttnCursor c;
      c.init(seqlens, B, seqlen_cap, k, first, count);
      long long n = 0;
      int ntile = 0;
      bool seg_first = true;
      while (c.valid() && !*abort_flag) {
        bool ok = true;
        // S = Q K^T over the nine 64-column chunks
        for (int cc = 0; cc < kAuQChunks && ok; ++cc, ++n) {
          const int slot = static_cast<int>(n % kAuSlots);
          ok = sm100::mbar_wait(&chunk_full[slot], static_cast<uint32_t>((n / kAuSlots) & 1));
          if (ok && cc == 0 && ntile > 0) ok = sm100::mbar_wait(pv_done, (ntile - 1) & 1);
          if (!ok) break;
          sm100::tc_fence_after();
          const uint32_t a0 = smem_u32(ring + slot * kAuSlotBytes);
          const uint32_t b0 = a0 + kAuQChunkBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            sm100::mma_bf16_ss(tm_s, sm100::smem_desc_k_sw128(a0 + 32 * kk), sm100::smem_desc_k_sw128(b0 + 32 * kk),
                               idesc_s, (cc | kk) != 0);
          sm100::mma_commit(&chunk_empty[slot]);
        }
        if (!ok) { *abort_flag = 1; break; }
        sm100::mma_commit(s_full);
        const int this_b = c.b;
        c.next(seqlens, B, seqlen_cap, k);
        const bool last_of_req = !c.valid() || c.b != this_b;
        // O += P V over this CTA's four value chunks
        if (!sm100::mbar_wait(p_full, ntile & 1)) { *abort_flag = 1; break; }
        sm100::tc_fence_after();
        for (int v = 0; v < kAuVChunks && ok; ++v, ++n) {
          const int slot = static_cast<int>(n % kAuSlots);
          ok = sm100::mbar_wait(&chunk_full[slot], static_cast<uint32_t>((n / kAuSlots) & 1));
          if (!ok) break;
          sm100::tc_fence_after();
          const uint32_t b0 = smem_u32(ring + slot * kAuSlotBytes + kAuQChunkBytes);
#pragma unroll
          for (int i = 0; i < kAuTile / 16; ++i)
            sm100::mma_bf16_ts(tm_o + 64 * v, tm_s + 8 * i,
                               sm100::smem_desc_mn_sw128(b0 + i * 2048, kAuChunkBytes, 1024), idesc_pv,
                               !(seg_first && i == 0));
          sm100::mma_commit(&chunk_empty[slot]);
        }
        if (!ok) { *abort_flag = 1; break; }
        sm100::mma_commit(pv_done);
        seg_first = last_of_req;
        ++ntile;
      }
    }
  }

  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  if (warp == 8) {
    __syncwarp();
    sm100::tmem_dealloc(tmem, 512);
  }
}

// Merges the per-range partials into the bf16 output. One block per (request,
// group of 8 heads): warp 0 finds the request's segments once (a request has
// at most ceil(k / 256) tiles, hence at most that many covering ranges: tile i
// of the list lies in range ((i + 1) * n_ranges - 1) / total), the (m, l) of
// 8 heads x those segments are staged in shared memory, and each thread merges
// 4 value columns of all 8 heads, its partial loads all in flight together.
constexpr int kAuMaxSeg = kMaxTopK / kAuTile;
constexpr int kAuCombineHeads = 8;

__global__ void __launch_bounds__(128) attn_mla_umma_combine_kernel(
    const float* __restrict__ part_o, const float2* __restrict__ part_ml, const int32_t* __restrict__ seqlens,
    int B, int k, int seqlen_cap, int n_ranges, __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  constexpr int HG = kAuHeads / kAuCombineHeads;
  const int b = blockIdx.x / HG;
  const int h0 = (blockIdx.x % HG) * kAuCombineHeads;
  __shared__ int seg_r[kAuMaxSeg];
  __shared__ float2 ml_s[kAuCombineHeads][kAuMaxSeg];
  const int tid = threadIdx.x, lane = tid & 31;
  if (tid < 32) {
    uint32_t before = 0, total = 0, mine = 0;
    for (int i = lane; i < B; i += 32) {
      int L = seqlens[i];
      L = L < 0 ? 0 : (L > seqlen_cap ? seqlen_cap : L);
      const uint32_t n = static_cast<uint32_t>(ceil_div(min(k, L), kAuTile));
      before += i < b ? n : 0;
      mine += i == b ? n : 0;
      total += n;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      before += __shfl_xor_sync(0xffffffffu, before, o);
      total += __shfl_xor_sync(0xffffffffu, total, o);
      mine += __shfl_xor_sync(0xffffffffu, mine, o);
    }
    const uint32_t nr = static_cast<uint32_t>(n_ranges);
    const uint32_t r = lane < static_cast<int>(mine) ? ((before + lane + 1) * nr - 1) / total : 0xffffffffu;
    const uint32_t prev = __shfl_up_sync(0xffffffffu, r, 1);
    if (lane < kAuMaxSeg) seg_r[lane] = (r != 0xffffffffu && (lane == 0 || r != prev)) ? static_cast<int>(r) : -1;
  }
  __syncthreads();
  if (tid < kAuCombineHeads * kAuMaxSeg) {
    const int hh = tid / kAuMaxSeg, j = tid % kAuMaxSeg;
    const int r = seg_r[j];
    ml_s[hh][j] = r >= 0 ? part_ml[((size_t)r + b) * kAuHeads + h0 + hh] : make_float2(-INFINITY, 0.f);
  }
  __syncthreads();
  const int d0 = 4 * tid;  // value columns d0..d0+3
  const int hf = d0 / (kAuDv / 2), dl = d0 % (kAuDv / 2);
#pragma unroll 2
  for (int hh = 0; hh < kAuCombineHeads; ++hh) {
    const int h = h0 + hh;
    float M = -INFINITY;
#pragma unroll
    for (int j = 0; j < kAuMaxSeg; ++j) M = fmaxf(M, ml_s[hh][j].x);
    float denom = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < kAuMaxSeg; ++j) {
      const float2 ml = ml_s[hh][j];
      if (ml.x == -INFINITY) continue;
      const size_t slot = static_cast<size_t>(seg_r[j]) + b;
      const float wgt = exp2f(ml.x - M);
      denom += wgt * ml.y;
      const float4 o = *reinterpret_cast<const float4*>(part_o + ((slot * 2 + hf) * kAuHeads + h) * (kAuDv / 2) + dl);
      acc.x += wgt * o.x;
      acc.y += wgt * o.y;
      acc.z += wgt * o.z;
      acc.w += wgt * o.w;
    }
    const float inv = denom > 0.f ? 1.f / denom : 0.f;
    __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(out + ((size_t)b * kAuHeads + h) * kAuDv + d0);
    o2[0] = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    o2[1] = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    if (lse != nullptr && tid == 0)
      lse[(size_t)b * kAuHeads + h] = denom > 0.f ? (M + log2f(denom)) * 0.69314718055994530942f : -INFINITY;
  }
}

inline size_t attn_umma_workspace(int B) {
  const size_t slots = static_cast<size_t>(kAuRanges) + B;
  const size_t o = slots * 2 * kAuHeads * (kAuDv / 2) * sizeof(float);
  return ((o + 255) / 256) * 256 + slots * kAuHeads * sizeof(float2);
}

}  // namespace sd
