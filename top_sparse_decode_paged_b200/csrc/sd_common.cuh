// Shared device helpers for the sparse decode kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sd_api.h"

namespace sd {

constexpr int kMaxTopK = 2048;  // largest k the library accepts

// Sticky per-device error word; kernels OR SD_DEVERR_* bits into it when
// device-resident data (seqlens, block tables, indices) is out of range.
__device__ unsigned int g_error_bits;

__device__ __forceinline__ void raise_error(unsigned int bit) { atomicOr(&g_error_bits, bit); }

// Timeline probes for tuning. Compiled out unless the library is built with
// -DSD_PROBE; then a mark stores the globaltimer (ns) into a fixed slot
// [kernel][block][event][index % 64] (a plain store: nothing waits on it),
// which sd_probe_read() copies out.
#ifdef SD_PROBE
constexpr int kProbeKernels = 4, kProbeBlocks = 1024, kProbeEvents = 16, kProbeIdx = 64;
__device__ unsigned long long g_probe[kProbeKernels][kProbeBlocks][kProbeEvents][kProbeIdx];
__device__ __forceinline__ void probe_mark(int kernel, int event, long long value) {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  const unsigned int blk = blockIdx.x + blockIdx.y * gridDim.x;
  if (kernel >= 1 && kernel <= kProbeKernels && blk < kProbeBlocks && event < kProbeEvents)
    g_probe[kernel - 1][blk][event][static_cast<unsigned int>(value) % kProbeIdx] = t;
}
#define SD_PROBE_MARK(k, e, v) ::sd::probe_mark((k), (e), (v))
#else
#define SD_PROBE_MARK(k, e, v) ((void)0)
#endif

// Clamp a device-resident sequence length to [0, cap]; flags the error bit.
__device__ __forceinline__ int checked_seqlen(const int32_t* seqlens, int b, int cap) {
  int L = seqlens[b];
  if (L < 0 || L > cap) {
    raise_error(SD_DEVERR_SEQLEN);
    L = L < 0 ? 0 : cap;
  }
  return L;
}

// Programmatic dependent launch. pdl_wait() blocks until the grids this one
// depends on in its stream have completed and their writes are visible; call
// it before reading anything earlier work produced. pdl_trigger() lets the
// next grid in the stream start launching (it still waits in pdl_wait()).
// Both are no-ops for a grid launched without the programmatic attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" :::); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Optional second output of the top-k: each selected token resolved to its
// pool row (page * page_size + slot) through the block table, [rows][kpad]
// with -1 for empty slots, so that the attention's gathers need no dependent
// block-table load. rows == nullptr disables it.
struct RowMap {
  int32_t* rows;
  const int32_t* block_table;
  int page_size, max_pages, num_pages, kpad;
  // `pcache` holds the last (block-table index, page) looked up by this
  // thread: a thread's selections are ascending and mostly share a page.
  __device__ __forceinline__ void put(int row, int b, int slot, int token, int2& pcache) const {
    if (rows == nullptr) return;
    int r = -1;
    if (token >= 0) {
      const int pi = token / page_size;
      if (pi != pcache.x) pcache = make_int2(pi, block_table[(size_t)b * max_pages + pi]);
      const int page = pcache.y;
      if (page >= 0 && page < num_pages) {
        r = page * page_size + token % page_size;
      } else {
        raise_error(SD_DEVERR_PAGE);
      }
    }
    rows[(size_t)row * kpad + slot] = r;
  }
  // The same for a token >= 0 whose block-table entry the caller loaded.
  __device__ __forceinline__ void put_page(int row, int slot, int token, int page) const {
    int r = -1;
    if (page >= 0 && page < num_pages) {
      r = page * page_size + token % page_size;
    } else {
      raise_error(SD_DEVERR_PAGE);
    }
    rows[(size_t)row * kpad + slot] = r;
  }
};

// 16-byte global->shared async copy; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async_16(void* smem_dst, const void* gmem_src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src), "r"(src_bytes)
               : "memory");
}
// 4-byte cp.async (through L1), for small index blocks of any alignment.
__device__ __forceinline__ void cp_async_4(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                            const void* smem_row_ptr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(smem_row_ptr)));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                                  const void* smem_row_ptr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(smem_row_ptr)));
}

// D += A(16x16 bf16, row) * B(16x8 bf16, col), fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace sd
