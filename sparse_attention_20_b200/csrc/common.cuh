// Shared device helpers of the DSA kernels (single translation unit: dsa.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dsa {

enum : int { kStatusOk = 0, kStatusTimeout = -4 };

// Device status word: kernels record the first failure here (never trap).
__device__ int g_status = 0;

// Where the first bounded wait gave up: {tag, chunk, block, parity}.
__device__ int g_timeout_info[4] = {0, 0, 0, 0};

__device__ __forceinline__ void report_status(int code) { atomicCAS(&g_status, 0, code); }

__device__ __forceinline__ void report_timeout(int tag, int chunk, int parity)
{
    if (atomicCAS(&g_status, 0, kStatusTimeout) == 0) {
        g_timeout_info[0] = tag;
        g_timeout_info[1] = chunk;
        g_timeout_info[2] = (int)blockIdx.x;
        g_timeout_info[3] = parity;
        __threadfence();
    }
}

// Order-preserving map fp32 -> uint32 (a > b  <=>  key(a) > key(b)); -0 is
// folded onto +0 so that equal scores compare equal.
__device__ __forceinline__ uint32_t score_key(float f)
{
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_score(uint32_t k)
{
    uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
    return __uint_as_float(u);
}

// Two e4m3 bytes (low byte first) -> two floats (exact: e4m3 is a subset of f16).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t v)
{
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(v));
    __half2 h = *reinterpret_cast<__half2*>(&h2);
    return __half22float2(h);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&b);
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the previous kernel on its stream is still
// running; it waits here, before its first read of global memory, until that
// kernel has completed and its writes are visible. (A no-op for a kernel
// launched without the attribute.)
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Candidate range of query row t: s = 0..n-1 at cache rows base + s. Rows that
// would reach outside the cache (a caller error) are clipped to it, so no
// kernel ever reads out of bounds.
__device__ __forceinline__ int row_candidates(const int* pos, const int* k_base, int t, int T,
                                              int S, long long* base_out)
{
    const long long base = k_base ? k_base[t] : 0;
    const long long p = pos ? pos[t] : (long long)t + S - T;
    *base_out = base;
    if (base < 0 || base >= S || p < 0) return 0;
    return (int)min(p + 1, (long long)S - base);
}

// A paged cache (serving form): logical key s of query row t lives at physical
// row block_table[seq[t] * max_pages + s / page_size] * page_size + s % page_size.
// block_table == NULL: keys are contiguous from k_base[t] (row_candidates).
struct PagedRows {
    const int* block_table = nullptr;
    const int* seq = nullptr;
    int n_seqs = 0, max_pages = 0, page_size = 1, num_pages = 0;
};

// Key count of row t; *base and *bt say where its keys live (key_row).
__device__ __forceinline__ int row_keys(const PagedRows& pg, const int* pos, const int* k_base, int t,
                                        int T, int S, long long* base, const int** bt)
{
    if (!pg.block_table) {
        *bt = nullptr;
        return row_candidates(pos, k_base, t, T, S, base);
    }
    *base = 0;
    const int sq = pg.seq[t];
    const long long p = pos[t];
    if (sq < 0 || sq >= pg.n_seqs || p < 0) {
        *bt = nullptr;
        return 0;
    }
    *bt = pg.block_table + (size_t)sq * pg.max_pages;
    return (int)min(p + 1, (long long)pg.max_pages * pg.page_size);
}

// Physical row of logical key s (0 <= s < row_keys). A block-table entry out
// of range reads page 0: wrong values, but no access outside the cache.
__device__ __forceinline__ long long key_row(const PagedRows& pg, const int* bt, long long base, int s)
{
    if (!bt) return base + s;
    int page = bt[s / pg.page_size];
    if ((unsigned)page >= (unsigned)pg.num_pages) page = 0;
    return (long long)page * pg.page_size + s % pg.page_size;
}

}  // namespace dsa
