// Sparse MLA decode attention on the 5th-generation tensor cores (tcgen05),
// for 128 query heads sharing one 576-wide latent row per token (V = the
// first 512 columns): the selected-token MLA of "Add DSA Vanilla sparse
// attention" (Walkthrough), consuming the top-k buffer of the DSA decode
// step ("Overlap DSA heuristic prev_topk write-back on the aux stream").
//
// Budget. The queries of one request (128 heads x 576 bf16) take 144 KB and
// its fp32 output (128 x 512) would fill all of tensor memory. So each tile
// range is served by two CTAs that split the heads, 64 each. A CTA keeps its
// 64 query heads resident (72 KB) and gathers every selected row of the range
// itself; the two CTAs of a range read the same rows at about the same time,
// so the second read is mostly an L2 hit.
//
// Per 64-token tile:
//   S   = Q K^T      M = 64 heads, N = 64 tokens, K = 576 (9 chunks of 64)
//   O^T += V^T P^T   M = 128 value rows (x4 blocks), N = 64 heads, K = 64 tokens
// Tensor memory: O^T in columns [0,256) (block j of 128 value rows at 64j),
// S double-buffered at [256,320) and [320,384) in the M = 64 layout (head
// 16 q + i in lane 32 q + i).
//
// Shared memory: Q (9 chunks x 64 heads x 128 B), two 72 KB tile buffers
// (9 chunks x 64 tokens x 128 B, the 128-byte swizzle), P^T (64 heads x 64
// tokens bf16), and a small ring of row ids. A tile chunk is the K-major B of
// S and, read MN-major, the A of O^T. Small-N MMAs are bound by reading their
// operands from shared memory, which is why S uses M = 64 (only real heads)
// and tiles are as wide as the buffers allow.
//
// Rows. Selections arrive resolved to pool rows (page * page_size + slot, -1
// to skip): the decode step's top-k writes them, a standalone call runs
// attn_rows_kernel. A warp streams each tile's 64 row ids into the ring a few
// tiles ahead, so no dependent block-table load sits on the gather's path.
// Gathers use coalesced cp.async: 8 lanes fetch one 128-byte row piece, the
// destination swizzle is applied per 16-byte lane, and skipped rows copy
// zeros. Measured on the part: scattered 1152-byte rows stream from HBM at
// about 3.1 TB/s by cp.async and 2.8 TB/s by 1-D bulk copies; pushing half of
// each tile to the partner CTA over distributed shared memory was slower than
// reading it twice through L2. Neither an L2 prefetch of upcoming rows nor
// staging the next tile in the copy threads' registers shortened the tile
// period.
//
// Softmax: a 16-lane tensor-memory load spreads each warp's 16 heads over all
// 32 threads (2 heads x 16 tokens each); max and sum are combined over the 4
// threads of a head with shuffles. The running max is updated lazily: O is
// rescaled only when a tile's max exceeds the reference by more than 2^8.
//
// Work: all requests' tiles (ceil(min(k, L) / 64) per request) form one list
// that is cut into equal contiguous ranges, one per CTA pair. A range that
// covers parts of several requests writes one partial (O, m, l) per request.
// The combine kernel merges them.
//
// Roles (352 threads): warps 0-3 copy (thread 0 also loads Q by TMA), warps
// 4-7 run the softmax, rescale and write partials (warp w owns TMEM lanes
// 32*(w%4)..+31), warp 8 owns tensor memory and issues the S products, warp
// 10 issues the P V products (each issuer blocks on its own inputs, in
// order), warp 9 streams row ids.
// Every wait is bounded (a timeout flags SD_DEVERR_TIMEOUT).
#pragma once

#include "sm100.cuh"

namespace sd {

constexpr int kAuTile = 64;                // selected tokens per tile
constexpr int kAuTileWords = kAuTile / 32; // 32-bit valid-token words per tile
constexpr int kAuHeads = 128;              // query heads of a request
constexpr int kAuHalfHeads = 64;           // query heads per CTA (M of S)
constexpr int kAuDk = 576, kAuDv = 512;
constexpr int kAuChunks = kAuDk / 64;      // 9 column chunks of 64
constexpr int kAuVBlocks = kAuDv / 128;    // 4 blocks of 128 value rows
constexpr int kAuChunkBytes = kAuTile * 128;              // 8 KB
constexpr int kAuTileBytes = kAuChunks * kAuChunkBytes;   // 72 KB
constexpr int kAuQChunkBytes = kAuHalfHeads * 128;        // 8 KB
constexpr int kAuQBytes = kAuChunks * kAuQChunkBytes;     // 72 KB
constexpr int kAuPChunk = kAuChunks - 1;  // P^T (64 heads x 64 tokens) goes into the tile's rope chunk once S is done
constexpr int kAuBufs = 2;
constexpr int kAuThreads = 352;
constexpr int kAuRidSlots = 4;             // row-id lookahead (tiles)
constexpr int kAuRanges = 74;              // CTA pairs: 148 CTAs, one per SM
constexpr float kAuRescaleLog2 = 8.0f;     // lazy rescale threshold (log2 units)
static_assert(kAuTile % 32 == 0 && kAuTile <= 64, "tile of 32 or 64 tokens");

// Row-id slots per request in the resolved-row array (whole tiles).
__host__ __device__ constexpr int attn_kpad(int k) { return (k + kAuTile - 1) / kAuTile * kAuTile; }

struct AttnUmmaLayout {
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = kOffQ + kAuQBytes;
  static constexpr int kOffBar = kOffRing + kAuBufs * kAuTileBytes;
  static constexpr int kNumBars = 4 * kAuBufs + 8 + 2 * kAuRidSlots;
  static constexpr int kOffRid = kOffBar + 8 * kNumBars;             // [slots][tile] pool row ids (-1: skip)
  static constexpr int kOffAlpha = kOffRid + 4 * kAuTile * kAuRidSlots;  // [64] rescale factors
  static constexpr int kOffMisc = kOffAlpha + 4 * kAuHalfHeads;
  static constexpr int kBytes = kOffMisc + 16;
  static constexpr size_t kSmemAlloc = kBytes + 1024;
};
static_assert(AttnUmmaLayout::kSmemAlloc <= 232448, "attention shared memory");

// Walks a contiguous range of the attention tile list (request-major).
// Requests are "virtual": vb = layer * breq + b when several layers share one
// selection (the row ids, seqlens and block table of request b), vb = b
// otherwise.
struct AttnCursor {
  int b, tile, tiles_b, L;
  long long remaining;
  int breq;
  __device__ static int tiles_of(int L, int k) { return ceil_div(min(k, L), kAuTile); }
  __device__ void init(const int32_t* seqlens, int B, int cap, int k, long long first, long long count, int nreq) {
    remaining = count;
    breq = nreq;
    long long skip = first;
    for (b = 0; b < B; ++b) {
      L = checked_seqlen(seqlens, b % breq, cap);
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
      L = checked_seqlen(seqlens, b % breq, cap);
      tiles_b = tiles_of(L, k);
    } while (tiles_b == 0 && b < B - 1);
  }
};

// Base pointers of the latent caches of the layers one launch serves.
constexpr int kAuMaxLayers = 16;
struct AttnLayerKV {
  const __nv_bfloat16* p[kAuMaxLayers];
};

__device__ __forceinline__ long long attn_total_tiles(const int32_t* seqlens, int B, int cap, int k, int breq) {
  long long n = 0;
  for (int b = 0; b < B; ++b) {
    int L = seqlens[b % breq];
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

// Resolves selections to pool rows for a standalone attention call (the
// decode step has the top-k write them): rows[b][s] for s < attn_kpad(k),
// -1 past min(k, L_b) and for skipped selections.
__global__ void __launch_bounds__(256) attn_rows_kernel(const int32_t* __restrict__ indices,
                                                        const int32_t* __restrict__ block_table,
                                                        const int32_t* __restrict__ seqlens, int k, int seqlen_cap,
                                                        int page_size, int max_pages, int num_pages,
                                                        int32_t* __restrict__ rows) {
  pdl_wait();  // inputs come from earlier work in the stream
  pdl_trigger();

  const int b = blockIdx.y;
  const int s = blockIdx.x * 256 + threadIdx.x;
  const int kpad = attn_kpad(k);
  if (s >= kpad) return;
  const int L = checked_seqlen(seqlens, b, seqlen_cap);
  rows[(size_t)b * kpad + s] = static_cast<int>(
      attn_row_of(indices, block_table, b, s, min(k, L), k, L, page_size, max_pages, num_pages));
}

// B counts virtual requests (layers x breq); q, out and the partials are
// indexed by them, seqlens and the row ids by the real request.
__global__ void __launch_bounds__(kAuThreads, 1) attn_mla_umma_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ AttnLayerKV kvl,
    const int32_t* __restrict__ seqlens, const int32_t* __restrict__ rows, int B, int breq, int k, int seqlen_cap,
    float scale_log2, float* __restrict__ part_o, float2* __restrict__ part_ml) {
  using Lay = AttnUmmaLayout;
  extern __shared__ uint8_t smem_dyn[];
  const uint32_t raw = smem_u32(smem_dyn);
  uint8_t* smem = smem_dyn + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* qbuf = smem + Lay::kOffQ;
  uint8_t* ring = smem + Lay::kOffRing;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kOffBar);
  uint64_t* tile_full = bars;                    // [bufs] 128 copy-thread arrivals (cp.async)
  uint64_t* tile_empty = bars + kAuBufs;         // [bufs] MMA commit after the tile's P V
  uint64_t* p_full = bars + 2 * kAuBufs;         // [bufs] the four softmax warps: P^T of the slot's tile written
  uint64_t* pv_done = bars + 3 * kAuBufs;        // [bufs] MMA commit after the slot's tile's P V
  uint64_t* q_full = bars + 4 * kAuBufs;         // 1 arrival + the Q bytes (TMA)
  uint64_t* q_empty = q_full + 1;                // MMA commit after a request's last S
  uint64_t* s_full = q_full + 2;                 // [2] MMA commit
  uint64_t* s_free = q_full + 4;                 // [2] the four softmax warps have read S
  uint64_t* mma_fin = q_full + 6;                // S issuer's commit at exit
  uint64_t* pv_fin = q_full + 7;                 // P V issuer's commit at exit
  uint64_t* rid_full = q_full + 8;               // [slots] 32 row-id lanes (cp.async)
  uint64_t* rid_empty = rid_full + kAuRidSlots;  // [slots] 4 copy warps + the epilogue
  int32_t* rid = reinterpret_cast<int32_t*>(smem + Lay::kOffRid);
  float* alpha_s = reinterpret_cast<float*>(smem + Lay::kOffAlpha);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_ranges = gridDim.x / 2;
  const int range = blockIdx.x % n_ranges;
  const int hh = blockIdx.x / n_ranges;  // which 64 query heads this CTA owns
  const int kpad = attn_kpad(k);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kAuBufs; ++i) {
      sm100::mbar_init(&tile_full[i], 128);
      sm100::mbar_init(&tile_empty[i], 1);
      sm100::mbar_init(&p_full[i], 4);
      sm100::mbar_init(&pv_done[i], 1);
    }
    sm100::mbar_init(q_full, 1);
    sm100::mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      sm100::mbar_init(&s_full[i], 1);
      sm100::mbar_init(&s_free[i], 4);
    }
    sm100::mbar_init(mma_fin, 1);
    sm100::mbar_init(pv_fin, 1);
    for (int i = 0; i < kAuRidSlots; ++i) {
      sm100::mbar_init(&rid_full[i], 32);
      sm100::mbar_init(&rid_empty[i], 5);
    }
    *abort_flag = 0;
    sm100::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) sm100::prefetch_tensormap(&tm_q);
  if (warp == 8) {
    sm100::tmem_alloc(tmem_slot, 512);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  // This range of the tile list follows from the sequence lengths alone. The
  // caller owns them and no kernel of the library writes them, so they are
  // read while the previous kernel may still be running; everything else
  // waits for it.
  const long long total = attn_total_tiles(seqlens, B, seqlen_cap, k, breq);
  const long long first = total * range / n_ranges;
  const long long count = total * (range + 1) / n_ranges - first;
  pdl_wait();
  pdl_trigger();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_o = tmem;          // cols [0,256): O^T, block j at 64j
  const uint32_t tm_s = tmem + 256;    // S, two buffers of kAuTile columns

  if (threadIdx.x == 0) SD_PROBE_MARK(3, 0, count);

  if (warp < 4) {
    // ------------------------------ copies ------------------------------
    // Thread pt fetches 16-byte column `seg` of tokens pt/8 + 16 i in all
    // nine chunks, so each copy instruction of a warp moves four 128-byte row
    // pieces.
    const int pt = threadIdx.x;  // 0..127
    const int seg = lane & 7;
    AttnCursor c;
    c.init(seqlens, B, seqlen_cap, k, first, count, breq);
    long long n = 0;
    int q_issued = 0, prev_b = -1;
    bool ok = true;
    while (c.valid() && ok) {
      if (c.b != prev_b) {
        // a new request: its 64 query heads into the Q buffer once the
        // previous request's S products are done with it
        prev_b = c.b;
        if (pt == 0) {
          if (q_issued > 0) ok = sm100::mbar_wait(q_empty, (q_issued - 1) & 1);
          if (ok) {
            sm100::mbar_arrive_expect_tx(q_full, kAuQBytes);
            for (int cc = 0; cc < kAuChunks; ++cc)
              sm100::tma_load_2d(qbuf + cc * kAuQChunkBytes, &tm_q, q_full, cc * 64,
                                 c.b * kAuHeads + hh * kAuHalfHeads);
            ++q_issued;
          } else {
            *abort_flag = 1;
          }
        }
      }
      const int rs = static_cast<int>(n % kAuRidSlots);
      ok = ok && sm100::mbar_wait(&rid_full[rs], static_cast<uint32_t>((n / kAuRidSlots) & 1));
      if (!ok) break;
      int row[kAuTile / 16];
#pragma unroll
      for (int i = 0; i < kAuTile / 16; ++i) row[i] = rid[rs * kAuTile + (pt >> 3) + 16 * i];
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&rid_empty[rs]);
      const int slot = static_cast<int>(n % kAuBufs);
      ok = ok && sm100::mbar_wait(&tile_empty[slot], static_cast<uint32_t>((n / kAuBufs) & 1) ^ 1) && !*abort_flag;
      if (!ok) break;
      uint8_t* tb = ring + slot * kAuTileBytes;
      const __nv_bfloat16* kv = kvl.p[c.b / breq];
#pragma unroll
      for (int i = 0; i < kAuTile / 16; ++i) {
        const int t = (pt >> 3) + 16 * i;
        const int rw = row[i];
        const __nv_bfloat16* src = kv + (long long)(rw >= 0 ? rw : 0) * kAuDk + seg * 8;
        uint8_t* dst = tb + t * 128 + ((seg ^ (t & 7)) << 4);
#pragma unroll
        for (int cc = 0; cc < kAuChunks; ++cc) cp_async_16(dst + cc * kAuChunkBytes, src + cc * 64, rw >= 0 ? 16 : 0);
      }
      sm100::cp_async_arrive_noinc(&tile_full[slot]);
      if (pt == 0) SD_PROBE_MARK(3, 1, n);
      ++n;
      c.next(seqlens, B, seqlen_cap, k);
    }
    cp_async_wait<0>();
    if (!ok) *abort_flag = 1;
    // the last Q load must have landed before the CTA exits
    if (pt == 0 && q_issued > 0) sm100::mbar_wait(q_full, (q_issued - 1) & 1);
  } else if (warp < 8) {
    // ------------------- softmax, rescale and partials -------------------
    // S is an M = 64 accumulator: head 16 q + i sits in TMEM lane 32 q + i
    // (i < 16). A 16-lane load spreads quadrant q's 16 heads over the warp:
    // thread t holds heads 16 q + t/4 and 16 q + t/4 + 8, 16 of the 64 tokens
    // each (tokens 8 r + 2 (t % 4) + {0, 1}); the 4 threads of a head combine
    // their max and sum with shuffles.
    constexpr int kReps = kAuTile / 8;  // 8-column repetitions of the 16x256b load
    const int quarter = warp & 3;
    const int tq = lane & 3;
    const int h0 = quarter * 16 + (lane >> 2);  // and h0 + 8
    const int vrow = quarter * 32 + lane;       // value row of O^T within a block
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    AttnCursor c;
    c.init(seqlens, B, seqlen_cap, k, first, count, breq);
    long long j = 0;
    int prev_b = -1;
    float m_ref[2] = {-INFINITY, -INFINITY}, l_sum[2] = {0.f, 0.f};
    while (c.valid()) {
      const bool seg_first = c.b != prev_b;
      prev_b = c.b;
      if (seg_first) {
        m_ref[0] = m_ref[1] = -INFINITY;
        l_sum[0] = l_sum[1] = 0.f;
      }
      const int rs = static_cast<int>(j % kAuRidSlots);
      uint32_t mask[kAuTileWords];
      bool ok = sm100::mbar_wait(&rid_full[rs], static_cast<uint32_t>((j / kAuRidSlots) & 1));
#pragma unroll
      for (int w = 0; w < kAuTileWords; ++w) mask[w] = __ballot_sync(0xffffffffu, rid[rs * kAuTile + 32 * w + lane] >= 0);
      ok = ok && sm100::mbar_wait(&s_full[j & 1], static_cast<uint32_t>((j >> 1) & 1)) && !*abort_flag;
      // one barrier makes the exit uniform and retires this tile's row-id slot
      ok = sm100::named_bar_and(1, 128, ok);
      if (!ok) { *abort_flag = 1; break; }
      if (threadIdx.x == 128) sm100::mbar_arrive(&rid_empty[rs]);
      if (threadIdx.x == 128) SD_PROBE_MARK(3, 6, j);
      sm100::tc_fence_after();
      uint32_t r[4 * kReps];
      sm100::tmem_ld_16x256b(tm_s + kAuTile * static_cast<uint32_t>(j & 1) + lane_base, r);
      sm100::tmem_ld_wait();
      if (threadIdx.x == 128) SD_PROBE_MARK(3, 7, j);
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&s_free[j & 1]);
      // valid bits of this thread's tokens 8 rr + 2 tq + {0, 1}
      uint32_t vb = 0;
#pragma unroll
      for (int rr = 0; rr < kReps; ++rr) {
        const int t0 = 8 * rr + 2 * tq;
        vb |= ((mask[t0 >> 5] >> (t0 & 31)) & 3u) << (2 * rr);
      }
      uint32_t pk[2][kReps];  // [head][rr]: bf16 pair of tokens 8 rr + 2 tq + {0, 1}
      bool need = false;
      // scaled logits (log2 units) of this thread's 2 heads x 2 kReps tokens;
      // skipped tokens are -inf, which the exponential maps to 0
      float y[2][2 * kReps];
#pragma unroll
      for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int q = 0; q < 2 * kReps; ++q)
          y[e][q] = ((vb >> q) & 1u) ? __uint_as_float(r[4 * (q >> 1) + 2 * e + (q & 1)]) * scale_log2 : -INFINITY;
      float mx[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float a[kReps];
#pragma unroll
        for (int i = 0; i < kReps; ++i) a[i] = fmaxf(y[e][2 * i], y[e][2 * i + 1]);
#pragma unroll
        for (int w2 = kReps / 2; w2 > 0; w2 >>= 1)
#pragma unroll
          for (int i = 0; i < w2; ++i) a[i] = fmaxf(a[i], a[i + w2]);
        mx[e] = a[0];
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 1));
#pragma unroll
      for (int e = 0; e < 2; ++e) mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 2));
      float m_use[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool ne = mx[e] > m_ref[e] + kAuRescaleLog2 || (m_ref[e] == -INFINITY && mx[e] > -INFINITY);
        float alpha = 1.f;
        if (ne) {
          alpha = exp2f(m_ref[e] - mx[e]);  // 0 when m_ref is -inf
          l_sum[e] *= alpha;
          m_ref[e] = mx[e];
        }
        need = need || ne;
        if (tq == 0) alpha_s[h0 + 8 * e] = alpha;
        m_use[e] = m_ref[e] == -INFINITY ? 0.f : m_ref[e];
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float l0 = 0.f, l1 = 0.f;
#pragma unroll
        for (int rr = 0; rr < kReps; ++rr) {
          const float p0 = sm100::ex2_approx(y[e][2 * rr] - m_use[e]);
          const float p1 = sm100::ex2_approx(y[e][2 * rr + 1] - m_use[e]);
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
          l0 += __low2float(h2);
          l1 += __high2float(h2);
          pk[e][rr] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        l_sum[e] += l0 + l1;
      }
      // earlier tiles of this request are in O: rescale when any head's
      // reference moved (alpha_s published by the barrier)
      const bool rescale = sm100::named_bar_or(2, 128, need && !seg_first);
      if (threadIdx.x == 128) SD_PROBE_MARK(3, 8, j);
      // P^T goes into this tile's rope chunk, which S has finished reading:
      // no wait. A rescale of O waits for the previous tile's P V first (each
      // slot's P V barrier is never waited more than one phase behind: the
      // slot's next P V needs a P^T not yet written).
      if (rescale && j > 0) {
        const long long jp = j - 1;
        bool okp = sm100::mbar_wait(&pv_done[jp % kAuBufs], static_cast<uint32_t>((jp / kAuBufs) & 1)) &&
                   !*abort_flag;
        okp = sm100::named_bar_and(3, 128, okp);
        if (!okp) { *abort_flag = 1; break; }
        sm100::tc_fence_after();
      }
      if (threadIdx.x == 128) SD_PROBE_MARK(3, 9, j);
      if (rescale) {
#pragma unroll 1
        for (int q8 = 0; q8 < 8; ++q8) {  // 4 value blocks x 2 halves of 32 head columns
          uint32_t ro[32];
          const uint32_t oa = tm_o + 32 * q8 + lane_base;
          sm100::tmem_ld_32x32b_x32(oa, ro);
          sm100::tmem_ld_wait();
          const float* al = alpha_s + 32 * (q8 & 1);
#pragma unroll
          for (int i = 0; i < 32; ++i) ro[i] = __float_as_uint(__uint_as_float(ro[i]) * al[i]);
          sm100::tmem_st_32x32b_x32(oa, ro);
        }
        sm100::tmem_st_wait();
      }
      {
        // P^T rows of heads h0, h0 + 8: this thread's 4-byte token pair in
        // each 16-byte piece, 128-byte swizzle
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int h = h0 + 8 * e;
          uint8_t* prow = ring + (j % kAuBufs) * kAuTileBytes + kAuPChunk * kAuChunkBytes + (h >> 3) * 1024 +
                          (h & 7) * 128 + 4 * tq;
#pragma unroll
          for (int rr = 0; rr < kReps; ++rr) *reinterpret_cast<uint32_t*>(prow + ((rr ^ (h & 7)) << 4)) = pk[e][rr];
        }
        sm100::fence_proxy_async_smem();
      }
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&p_full[j % kAuBufs]);
      if (threadIdx.x == 128) SD_PROBE_MARK(3, 3, j);
      if (lane == 0 && warp > 4) SD_PROBE_MARK(3, 5 + warp, j);  // events 10-12: the other warps' P

      const int this_b = c.b;
      c.next(seqlens, B, seqlen_cap, k);
      const bool seg_last = !c.valid() || c.b != this_b;
      if (seg_last) {
        bool okd = sm100::mbar_wait(&pv_done[j % kAuBufs], static_cast<uint32_t>((j / kAuBufs) & 1)) && !*abort_flag;
        okd = sm100::named_bar_and(4, 128, okd);
        if (!okd) { *abort_flag = 1; break; }
        sm100::tc_fence_after();
        const size_t slot = static_cast<size_t>(range) + this_b;
        float* dst = part_o + (slot * kAuHeads + hh * kAuHalfHeads) * kAuDv + vrow;
#pragma unroll 1
        for (int q8 = 0; q8 < 8; ++q8) {  // block q8/2, head columns 32*(q8%2)..+31
          uint32_t ro[32];
          sm100::tmem_ld_32x32b_x32(tm_o + 32 * q8 + lane_base, ro);
          sm100::tmem_ld_wait();
          float* d = dst + (q8 >> 1) * 128 + (size_t)(32 * (q8 & 1)) * kAuDv;
#pragma unroll
          for (int i = 0; i < 32; ++i) d[(size_t)i * kAuDv] = __uint_as_float(ro[i]);
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float l = l_sum[e];
          l += __shfl_xor_sync(0xffffffffu, l, 1);
          l += __shfl_xor_sync(0xffffffffu, l, 2);
          if (tq == 0) part_ml[slot * kAuHeads + hh * kAuHalfHeads + h0 + 8 * e] = make_float2(m_ref[e], l);
        }
        sm100::tc_fence_before();
      }
      ++j;
    }
  } else if (warp == 8) {
    // ------------------------------ S issue ------------------------------
    // S(i) needs tile i landed (and its request's Q) and S buffer i % 2 read
    // out by the softmax. A second thread (warp 10) issues the P V products,
    // so that neither kind waits behind the other's inputs; each issuer
    // blocks on its own barriers in order.
    if (sm100::elect_one()) {
      constexpr uint32_t idesc_s = sm100::idesc_bf16(kAuHalfHeads, kAuTile, false, false);
      const uint32_t qa = smem_u32(qbuf);
      AttnCursor cs;
      cs.init(seqlens, B, seqlen_cap, k, first, count, breq);
      int q_seen = 0, prev_bs = -1;
      bool ok = true;
      for (long long is = 0; is < count && ok; ++is) {
        const bool seg_first = cs.b != prev_bs;
        const int slot = static_cast<int>(is % kAuBufs);
        const int sb = static_cast<int>(is & 1);
        ok = (!seg_first || sm100::mbar_wait(q_full, static_cast<uint32_t>(q_seen & 1))) &&
             sm100::mbar_wait(&tile_full[slot], static_cast<uint32_t>((is / kAuBufs) & 1)) &&
             (is < 2 || sm100::mbar_wait(&s_free[sb], static_cast<uint32_t>(((is - 2) >> 1) & 1))) && !*abort_flag;
        if (!ok) break;
        sm100::tc_fence_after();
        if (seg_first) ++q_seen;
        prev_bs = cs.b;
        // S = Q K^T (M = 64 heads) over the nine 64-column chunks
        const uint32_t ta = smem_u32(ring + slot * kAuTileBytes);
#pragma unroll
        for (int cc = 0; cc < kAuChunks; ++cc)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            sm100::mma_bf16_ss(tm_s + kAuTile * sb, sm100::smem_desc_k_sw128(qa + cc * kAuQChunkBytes + 32 * kk),
                               sm100::smem_desc_k_sw128(ta + cc * kAuChunkBytes + 32 * kk), idesc_s,
                               (cc | kk) != 0);
        sm100::mma_commit(&s_full[sb]);
        SD_PROBE_MARK(3, 2, is);
        const int this_b = cs.b;
        cs.next(seqlens, B, seqlen_cap, k);
        if (is + 1 >= count || cs.b != this_b) sm100::mma_commit(q_empty);
      }
      if (!ok) *abort_flag = 1;
      // every issued MMA completes before tensor memory is released
      sm100::mma_commit(mma_fin);
      sm100::mbar_wait(mma_fin, 0);
    }
  } else if (warp == 10) {
    // ----------------------------- P V issue -----------------------------
    // P V(j) needs P(j) written (which follows S(j) and P V(j - 1)).
    if (sm100::elect_one()) {
      constexpr uint32_t idesc_pv = sm100::idesc_bf16(128, kAuHalfHeads, true, false);
      AttnCursor cp;
      cp.init(seqlens, B, seqlen_cap, k, first, count, breq);
      int prev_bp = -1;
      bool ok = true;
      for (long long ip = 0; ip < count && ok; ++ip) {
        ok = sm100::mbar_wait(&p_full[ip % kAuBufs], static_cast<uint32_t>((ip / kAuBufs) & 1)) && !*abort_flag;
        if (!ok) break;
        SD_PROBE_MARK(3, 13, ip);
        sm100::tc_fence_after();
        const bool seg_first = cp.b != prev_bp;
        prev_bp = cp.b;
        const int slot = static_cast<int>(ip % kAuBufs);
        const uint32_t ta = smem_u32(ring + slot * kAuTileBytes);
        const uint32_t pa = ta + kAuPChunk * kAuChunkBytes;
        // O^T += V^T P^T (chunks 2v, 2v+1 are value block v)
#pragma unroll
        for (int v = 0; v < kAuVBlocks; ++v)
#pragma unroll
          for (int kk = 0; kk < kAuTile / 16; ++kk)
            sm100::mma_bf16_ss(tm_o + 64 * v,
                               sm100::smem_desc_mn_sw128(ta + 2 * v * kAuChunkBytes + kk * 2048, kAuChunkBytes, 1024),
                               sm100::smem_desc_k_sw128(pa + 32 * kk), idesc_pv, !(seg_first && kk == 0));
        sm100::mma_commit(&tile_empty[slot]);
        sm100::mma_commit(&pv_done[slot]);
        SD_PROBE_MARK(3, 4, ip);
        cp.next(seqlens, B, seqlen_cap, k);
      }
      if (!ok) *abort_flag = 1;
      sm100::mma_commit(pv_fin);
      sm100::mbar_wait(pv_fin, 0);
    }
  } else if (warp == 9) {
    // ------------------------------ row ids ------------------------------
    // Streams each tile's resolved pool rows into a small ring, kAuRidSlots
    // tiles ahead of the copies and the softmax.
    AttnCursor c;
    c.init(seqlens, B, seqlen_cap, k, first, count, breq);
    long long n = 0;
    bool ok = true;
    while (c.valid() && ok) {
      const int rs = static_cast<int>(n % kAuRidSlots);
      ok = sm100::mbar_wait(&rid_empty[rs], static_cast<uint32_t>((n / kAuRidSlots) & 1) ^ 1) && !*abort_flag;
      if (!ok) break;
      const int32_t* src = rows + (size_t)(c.b % breq) * kpad + c.tile * kAuTile;
#pragma unroll
      for (int w = 0; w < kAuTileWords; ++w) cp_async_4(&rid[rs * kAuTile + 32 * w + lane], src + 32 * w + lane);
      sm100::cp_async_arrive_noinc(&rid_full[rs]);
      ++n;
      c.next(seqlens, B, seqlen_cap, k);
    }
    cp_async_wait<0>();
    if (!ok) *abort_flag = 1;
  }

  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  if (threadIdx.x == 0) SD_PROBE_MARK(3, 5, 0);
  if (warp == 8) {
    __syncwarp();
    sm100::tmem_dealloc(tmem, 512);
  }
}

// Merges the per-range partials into the bf16 output: one warp per (request,
// head), 16 heads per block, one wave. The ranges that cover a request follow
// from the tile list in closed form: tile i lies in range ((i + 1) *
// n_ranges - 1) / total, so with total >= n_ranges a request's tiles
// [t0, t0 + n) span the consecutive ranges range(t0) .. range(t0 + n - 1),
// and with fewer tiles than ranges each tile has a range of its own. Lane s
// loads the (m, l) of segments s and s + 32 for the head; each lane then
// merges 16 contiguous value columns over the segments.
constexpr int kAuMaxSeg = kMaxTopK / kAuTile;
constexpr int kAuCombineHeads = 16;  // heads (warps) per block
constexpr int kAuSegPerLane = (kAuMaxSeg + 31) / 32;

__global__ void __launch_bounds__(32 * kAuCombineHeads, 2) attn_mla_umma_combine_kernel(
    const float* __restrict__ part_o, const float2* __restrict__ part_ml, const int32_t* __restrict__ seqlens,
    int B, int breq, int k, int seqlen_cap, int n_ranges, __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  constexpr int HG = kAuHeads / kAuCombineHeads;
  const int b = blockIdx.x / HG;
  const int h = (blockIdx.x % HG) * kAuCombineHeads + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  uint32_t before = 0, total = 0, mine = 0;
  for (int i = lane; i < B; i += 32) {
    int L = seqlens[i % breq];
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
  const unsigned long long nr = static_cast<unsigned long long>(n_ranges);
  auto range_of = [&](uint32_t i) { return static_cast<uint32_t>(((i + 1ull) * nr - 1ull) / total); };
  uint32_t nseg = 0, r0 = 0;
  if (mine > 0) {
    r0 = range_of(before);
    nseg = total >= nr ? range_of(before + mine - 1) - r0 + 1 : mine;
  }
  auto seg_range = [&](uint32_t sg) { return total >= nr ? r0 + sg : range_of(before + sg); };
  // The segments above follow from the caller's sequence lengths, which no
  // kernel of the library writes; the partials come from the attention.
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0 && (blockIdx.x & 15) == 0) SD_PROBE_MARK(4, 0, 0);
  // a segment's 16 values of this lane's columns (zeros past the last one):
  // every written partial is finite, so rows of zero weight add nothing
  auto load_seg = [&](uint32_t sg, float4 (&v)[4]) {
    if (sg < nseg) {
      const float4* src = reinterpret_cast<const float4*>(
          part_o + (((size_t)seg_range(sg) + b) * kAuHeads + h) * kAuDv + 16 * lane);
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = src[i];
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  // the first segment's row loads together with every segment's (m, l): it
  // does not depend on the weights
  float4 v0[4];
  load_seg(0, v0);
  float2 ml[kAuSegPerLane];
  float M = -INFINITY;
#pragma unroll
  for (int q = 0; q < kAuSegPerLane; ++q) {
    const uint32_t sg = static_cast<uint32_t>(lane + 32 * q);
    ml[q] = sg < nseg ? part_ml[((size_t)seg_range(sg) + b) * kAuHeads + h] : make_float2(-INFINITY, 0.f);
    M = fmaxf(M, ml[q].x);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float wgt[kAuSegPerLane], denom = 0.f;
#pragma unroll
  for (int q = 0; q < kAuSegPerLane; ++q) {
    wgt[q] = ml[q].x == -INFINITY ? 0.f : exp2f(ml[q].x - M);
    denom += wgt[q] * ml[q].y;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) denom += __shfl_xor_sync(0xffffffffu, denom, o);
  auto weight_of = [&](uint32_t sg) {
    float wq = wgt[0];
#pragma unroll
    for (int q = 1; q < kAuSegPerLane; ++q)
      if ((sg >> 5) == static_cast<uint32_t>(q)) wq = wgt[q];
    const float ws = __shfl_sync(0xffffffffu, wq, static_cast<int>(sg & 31));
    return sg < nseg ? ws : 0.f;
  };
  float acc[16];
  {
    const float w0 = weight_of(0);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[4 * i] = w0 * v0[i].x;
      acc[4 * i + 1] = w0 * v0[i].y;
      acc[4 * i + 2] = w0 * v0[i].z;
      acc[4 * i + 3] = w0 * v0[i].w;
    }
  }
  // the other segments two at a time
  for (uint32_t s0 = 1; s0 < nseg; s0 += 2) {
    float4 v[2][4];
    load_seg(s0, v[0]);
    load_seg(s0 + 1, v[1]);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float ws = weight_of(s0 + u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[4 * i] += ws * v[u][i].x;
        acc[4 * i + 1] += ws * v[u][i].y;
        acc[4 * i + 2] += ws * v[u][i].z;
        acc[4 * i + 3] += ws * v[u][i].w;
      }
    }
  }
  const float inv = denom > 0.f ? 1.f / denom : 0.f;
  uint32_t pk[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(acc[2 * i] * inv, acc[2 * i + 1] * inv);
  uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)b * kAuHeads + h) * kAuDv + 16 * lane);
  dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  if (lse != nullptr && lane == 0)
    lse[(size_t)b * kAuHeads + h] = denom > 0.f ? (M + log2f(denom)) * 0.69314718055994530942f : -INFINITY;
  if (threadIdx.x == 0 && (blockIdx.x & 15) == 0) SD_PROBE_MARK(4, 1, 0);
}

// Workspace: partial O [slots][128][512] fp32, (m, l) [slots][128], and the
// resolved row ids [B][attn_kpad(k)] int32.
inline size_t attn_umma_rows_offset(int B) {
  const size_t slots = static_cast<size_t>(kAuRanges) + B;
  const size_t o = ((slots * kAuHeads * kAuDv * sizeof(float) + 255) / 256) * 256;
  return o + ((slots * kAuHeads * sizeof(float2) + 255) / 256) * 256;
}
inline size_t attn_umma_workspace(int B, int k) {
  return attn_umma_rows_offset(B) + static_cast<size_t>(B) * attn_kpad(k) * sizeof(int32_t);
}

}  // namespace sd
