// Sparse attention over selected paged rows, split over the selected set,
// followed by a combine pass (warp-level mma.sync path, all head geometries).
//
// For each query head h of KV head g (contiguous groups) and its selected
// request-local tokens j:  o = sum_j softmax_j(scale * q . K_j) V_j, with K_j,
// V_j gathered through the block table. This is the "core sparse attention"
// that consumes the top-k buffer ("Overlap DSA heuristic prev_topk
// write-back...", Description) over a paged latent cache ("Add DSA Vanilla
// sparse attention", Walkthrough: selected-token MLA over NHD latent caches).
//
// Work split: one CTA per (request, KV head, block of HB query heads, split of
// the k index slots). Each CTA first resolves all of its slots to pool rows
// (index load, then block-table load: every thread's lookups in flight
// together, into shared memory), then streams its slots in tiles of 64 rows,
// gathered with cp.async into padded shared rows (double buffered), so no
// dependent lookup sits between two tiles. Per tile:
//   S = Q K^T on tensor cores (warps split the 64 tokens), an online softmax
//   whose row maxima and sums are shared through shared memory, P written to
//   shared memory as bf16, then O += P V (warps split the value columns).
// The CTA writes its unnormalised O with (m, l) in the log2 domain; the
// combine kernel merges the splits and rounds to bf16 (nearest even).
#pragma once

#include "sd_common.cuh"

namespace sd {

constexpr int kAttnTile = 64;  // selected rows per tile

template <int DK, int DV, int MT>
struct AttnMmaCfg {
  static constexpr int HB = 16 * MT;          // query heads per CTA
  static constexpr int WARPS = 4 * MT;
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int KS = DK + 8;           // padded smem row (elements)
  static constexpr int VS = DV + 8;
  static constexpr int PS = kAttnTile + 8;
  static constexpr int DV_PER_WARP = DV / 4;  // value columns per warp
  static constexpr int NV8 = DV_PER_WARP / 8; // n8 tiles per warp in P.V
  // shared memory for a split of `slots` index slots
  static size_t smem_bytes(bool separate_v, int slots) {
    size_t s = sizeof(long long) * ((slots + kAttnTile - 1) / kAttnTile) * kAttnTile;  // resolved rows
    s += sizeof(__nv_bfloat16) * HB * KS;                        // Q
    s += sizeof(__nv_bfloat16) * 2 * kAttnTile * KS;             // K tiles
    if (separate_v) s += sizeof(__nv_bfloat16) * 2 * kAttnTile * VS;  // V tiles
    s += sizeof(__nv_bfloat16) * HB * PS;                        // P
    s += sizeof(float) * 2 * 4 * HB;                             // row max / sum partials
    return s;
  }
};

template <int DK, int DV, int MT>
__global__ void __launch_bounds__(AttnMmaCfg<DK, DV, MT>::THREADS) attn_split_mma_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k_pages,
    const __nv_bfloat16* __restrict__ v_pages, const int32_t* __restrict__ block_table,
    const int32_t* __restrict__ seqlens, const int32_t* __restrict__ indices, int num_pages,
    int page_size, int max_pages, int G, int H, int k, int seqlen_cap, float scale_log2,
    int n_head_blocks, int n_splits, int slots_per_split, float* __restrict__ part_o,
    float2* __restrict__ part_ml) {
  pdl_wait();  // inputs come from earlier work in the stream
  pdl_trigger();

  using C = AttnMmaCfg<DK, DV, MT>;
  constexpr int HB = C::HB, KS = C::KS, VS = C::VS, PS = C::PS;
  const bool separate_v = v_pages != nullptr;

  extern __shared__ __align__(16) unsigned char smem_raw[];
  long long* sRow = reinterpret_cast<long long*>(smem_raw);  // the split's resolved pool rows (-1: skip)
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(
      smem_raw + sizeof(long long) * ((slots_per_split + kAttnTile - 1) / kAttnTile) * kAttnTile);
  __nv_bfloat16* sK = sQ + HB * KS;
  __nv_bfloat16* sV = sK + 2 * kAttnTile * KS;
  __nv_bfloat16* sP = separate_v ? sV + 2 * kAttnTile * VS : sV;
  float* sMax = reinterpret_cast<float*>(sP + HB * PS);
  float* sSum = sMax + 4 * HB;

  const int split = blockIdx.x;
  const int hb = blockIdx.y;
  const int bg = blockIdx.z;  // b * G + g
  const int b = bg / G, g = bg % G;
  const int qpk = H / G;
  const int h0 = g * qpk + hb * HB;               // first query head of this CTA
  const int nh = min(HB, qpk - hb * HB);          // valid heads in this block
  const int L = checked_seqlen(seqlens, b, seqlen_cap);
  const int slot0 = split * slots_per_split;
  const int slot1 = min(min(k, L), slot0 + slots_per_split);  // only the first min(k, L) slots are read
  const int ntiles = slot1 > slot0 ? ceil_div(slot1 - slot0, kAttnTile) : 0;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int mt = warp >> 2;   // m16 tile of this warp
  const int wq = warp & 3;    // token quarter (S) / value quarter (P.V)

  // Q rows (zero for padding heads)
  for (int c = tid; c < HB * (DK / 8); c += C::THREADS) {
    const int r = c / (DK / 8), ch = c % (DK / 8);
    const bool ok = r < nh;
    const __nv_bfloat16* src = q + ((size_t)b * H + h0 + (ok ? r : 0)) * DK + ch * 8;
    cp_async_16(sQ + r * KS + ch * 8, src, ok ? 16 : 0);
  }
  cp_async_commit();

  // every slot of the split resolved to its pool row, lookups in flight together
  const int32_t* idx_row = indices + (size_t)bg * k;
  for (int i = tid; i < ntiles * kAttnTile; i += C::THREADS) {
    const int slot = slot0 + i;
    long long rid = -1;
    if (slot < slot1) {
      const int t = idx_row[slot];
      if (t >= 0) {
        if (t >= L) {
          raise_error(SD_DEVERR_INDEX);
        } else {
          const int page = block_table[(size_t)b * max_pages + t / page_size];
          if (page < 0 || page >= num_pages) {
            raise_error(SD_DEVERR_PAGE);
          } else {
            rid = ((long long)page * page_size + (t % page_size)) * G + g;
          }
        }
      }
    }
    sRow[i] = rid;
  }
  __syncthreads();
  auto issue_copy = [&](int tile, int buf) {
    for (int c = tid; c < kAttnTile * (DK / 8); c += C::THREADS) {
      const int r = c / (DK / 8), ch = c % (DK / 8);
      const long long rid = sRow[tile * kAttnTile + r];
      const __nv_bfloat16* src = k_pages + (rid >= 0 ? rid : 0) * DK + ch * 8;
      cp_async_16(sK + (buf * kAttnTile + r) * KS + ch * 8, src, rid >= 0 ? 16 : 0);
    }
    if (separate_v) {
      for (int c = tid; c < kAttnTile * (DV / 8); c += C::THREADS) {
        const int r = c / (DV / 8), ch = c % (DV / 8);
        const long long rid = sRow[tile * kAttnTile + r];
        const __nv_bfloat16* src = v_pages + (rid >= 0 ? rid : 0) * DV + ch * 8;
        cp_async_16(sV + (buf * kAttnTile + r) * VS + ch * 8, src, rid >= 0 ? 16 : 0);
      }
    }
  };

  // per-thread softmax state for rows (lane/4) and (lane/4 + 8) of its m-tile
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  float o_acc[C::NV8][4];
#pragma unroll
  for (int i = 0; i < C::NV8; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.f;

  if (ntiles > 0) {
    issue_copy(0, 0);
    cp_async_commit();
  }
  for (int tile = 0; tile < ntiles; ++tile) {
    const int buf = tile & 1, nb = buf ^ 1;
    if (tile + 1 < ntiles) {
      issue_copy(tile + 1, nb);  // buffer nb (tile - 1) was released by the last barrier of that tile
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();

    const __nv_bfloat16* kt = sK + buf * kAttnTile * KS;
    const __nv_bfloat16* vt = separate_v ? sV + buf * kAttnTile * VS : kt;
    const int vstride = separate_v ? VS : KS;

    // ---- S = Q K^T for this warp's 16 heads x 16 tokens ----
    float s_acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 4
    for (int kk = 0; kk < DK / 16; ++kk) {
      uint32_t a[4];
      const __nv_bfloat16* qa = sQ + (mt * 16 + (lane & 15)) * KS + kk * 16 + (lane >> 4) * 8;
      ldmatrix_x4(a[0], a[1], a[2], a[3], qa);
      uint32_t b0, b1, b2, b3;
      // matrices: (tok 0-7, k 0-7), (tok 0-7, k 8-15), (tok 8-15, k 0-7), (tok 8-15, k 8-15)
      const int trow = wq * 16 + (lane & 7) + ((lane >> 4) << 3);
      const __nv_bfloat16* kb = kt + trow * KS + kk * 16 + ((lane >> 3) & 1) * 8;
      ldmatrix_x4(b0, b1, b2, b3, kb);
      mma_bf16_16816(s_acc[0], a, b0, b1);
      mma_bf16_16816(s_acc[1], a, b2, b3);
    }

    // ---- online softmax across the 4 token quarters ----
    const long long* rows = sRow + tile * kAttnTile;
    float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = wq * 16 + nt * 8 + 2 * (lane & 3) + (e & 1);
        const float z = rows[tok] >= 0 ? s_acc[nt][e] * scale_log2 : -INFINITY;
        s_acc[nt][e] = z;
        tmax[e >> 1] = fmaxf(tmax[e >> 1], z);
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 1));
      tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 2));
    }
    if ((lane & 3) == 0) {
      sMax[wq * HB + mt * 16 + (lane >> 2)] = tmax[0];
      sMax[wq * HB + mt * 16 + (lane >> 2) + 8] = tmax[1];
    }
    __syncthreads();
    float m_new[2], m_use[2], alpha[2], psum[2] = {0.f, 0.f};
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int row = mt * 16 + (lane >> 2) + 8 * r;
      float mx = m_run[r];
#pragma unroll
      for (int j = 0; j < 4; ++j) mx = fmaxf(mx, sMax[j * HB + row]);
      m_new[r] = mx;
      m_use[r] = mx == -INFINITY ? 0.f : mx;
      alpha[r] = exp2f(m_run[r] - m_use[r]);
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const float p0 = exp2f(s_acc[nt][0] - m_use[0]);
      const float p1 = exp2f(s_acc[nt][1] - m_use[0]);
      const float p2 = exp2f(s_acc[nt][2] - m_use[1]);
      const float p3 = exp2f(s_acc[nt][3] - m_use[1]);
      psum[0] += p0 + p1;
      psum[1] += p2 + p3;
      const int col = wq * 16 + nt * 8 + 2 * (lane & 3);
      const int row = mt * 16 + (lane >> 2);
      *reinterpret_cast<uint32_t*>(sP + row * PS + col) = pack_bf16x2(p0, p1);
      *reinterpret_cast<uint32_t*>(sP + (row + 8) * PS + col) = pack_bf16x2(p2, p3);
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      psum[r] += __shfl_xor_sync(0xffffffffu, psum[r], 1);
      psum[r] += __shfl_xor_sync(0xffffffffu, psum[r], 2);
    }
    if ((lane & 3) == 0) {
      sSum[wq * HB + mt * 16 + (lane >> 2)] = psum[0];
      sSum[wq * HB + mt * 16 + (lane >> 2) + 8] = psum[1];
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int row = mt * 16 + (lane >> 2) + 8 * r;
      float ts = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) ts += sSum[j * HB + row];
      l_run[r] = l_run[r] * alpha[r] + ts;
      m_run[r] = m_new[r];
    }

    // ---- O = O * alpha + P V over this warp's value columns ----
#pragma unroll
    for (int i = 0; i < C::NV8; ++i) {
      o_acc[i][0] *= alpha[0];
      o_acc[i][1] *= alpha[0];
      o_acc[i][2] *= alpha[1];
      o_acc[i][3] *= alpha[1];
    }
#pragma unroll
    for (int kk = 0; kk < kAttnTile / 16; ++kk) {
      uint32_t a[4];
      const __nv_bfloat16* pa = sP + (mt * 16 + (lane & 15)) * PS + kk * 16 + (lane >> 4) * 8;
      ldmatrix_x4(a[0], a[1], a[2], a[3], pa);
#pragma unroll
      for (int i = 0; i < C::NV8; i += 2) {
        // matrices: (tok 0-7, n 0-7), (tok 8-15, n 0-7), (tok 0-7, n 8-15), (tok 8-15, n 8-15)
        const int tok = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int col = wq * C::DV_PER_WARP + i * 8 + (lane >> 4) * 8;
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(b0, b1, b2, b3, vt + tok * vstride + col);
        mma_bf16_16816(o_acc[i], a, b0, b1);
        mma_bf16_16816(o_acc[i + 1], a, b2, b3);
      }
    }
    __syncthreads();  // sP, sMax, sSum and this buffer are rewritten next tile
  }

  cp_async_wait<0>();

  // ---- write the split partial ----
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = mt * 16 + (lane >> 2) + 8 * r;
    if (row >= nh) continue;
    const size_t pidx = ((size_t)b * H + h0 + row) * n_splits + split;
    if (wq == 0 && (lane & 3) == 0) part_ml[pidx] = make_float2(m_run[r], l_run[r]);
    float* dst = part_o + pidx * DV + wq * C::DV_PER_WARP + 2 * (lane & 3);
#pragma unroll
    for (int i = 0; i < C::NV8; ++i)
      *reinterpret_cast<float2*>(dst + i * 8) = make_float2(o_acc[i][2 * r], o_acc[i][2 * r + 1]);
  }
}

// Merge the splits of one (request, head): O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
template <int DV>
__global__ void __launch_bounds__(128) attn_combine_kernel(const float* __restrict__ part_o,
                                                           const float2* __restrict__ part_ml,
                                                           int n_splits, __nv_bfloat16* __restrict__ out,
                                                           float* __restrict__ lse) {
  pdl_wait();  // inputs come from earlier work in the stream
  pdl_trigger();

  const int bh = blockIdx.x;
  const float2* ml = part_ml + (size_t)bh * n_splits;
  float M = -INFINITY;
  for (int s = 0; s < n_splits; ++s) M = fmaxf(M, ml[s].x);
  float denom = 0.f;
  for (int s = 0; s < n_splits; ++s)
    if (ml[s].x != -INFINITY) denom += exp2f(ml[s].x - M) * ml[s].y;
  const float inv = denom > 0.f ? 1.f / denom : 0.f;
  for (int d = threadIdx.x; d < DV; d += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < n_splits; ++s)
      if (ml[s].x != -INFINITY) acc += exp2f(ml[s].x - M) * part_o[((size_t)bh * n_splits + s) * DV + d];
    out[(size_t)bh * DV + d] = __float2bfloat16_rn(acc * inv);
  }
  if (lse != nullptr && threadIdx.x == 0)
    lse[bh] = denom > 0.f ? (M + log2f(denom)) * 0.69314718055994530942f : -INFINITY;
}

}  // namespace sd
