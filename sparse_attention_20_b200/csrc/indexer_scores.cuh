// Lightning-indexer scores of a block of query rows against their causal key
// ranges, written to a row-major score buffer (one row per query row).
//
//   I_{t,s} = sum_{j<H_I} w_{t,j} * ReLU(q^I_{t,j} . k^I_s)
//   ("Paper Breakdown: DeepSeek-V3.2", section 2, "Index score")
//
// The contraction over d_I runs on the tensor cores as mma.sync m16n8k32
// (e4m3 x e4m3 -> fp32): 16 keys (A rows) against 8 heads (B columns) per
// instruction. The scan is HBM-bound (d_I bytes per key and ~2 flops per
// byte per head), so the legacy warp-level MMA is ample here; what matters is
// streaming the key rows with wide loads.
//
// Each thread owns d_I/4 contiguous bytes of a key row (its "quarter"); k-step
// kk of the MMA takes bytes [8kk, 8kk+8) of every quarter, and the query
// fragment uses the same byte permutation, so A and B agree on which d each
// MMA slot holds.
#pragma once
#include "common.cuh"

namespace dsa {

template <int DI>
struct KeyQuarter {
    static constexpr int kBytes = DI / 4;    // bytes per thread per key row
    static constexpr int kWords = kBytes / 4;
    uint32_t v[kWords];
    __device__ __forceinline__ void load(const uint8_t* p)
    {
        if constexpr (kBytes >= 16) {
#pragma unroll
            for (int i = 0; i < kBytes / 16; ++i) {
                uint4 x = __ldg(reinterpret_cast<const uint4*>(p) + i);
                v[4 * i + 0] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
            }
        } else {
            uint2 x = __ldg(reinterpret_cast<const uint2*>(p));
            v[0] = x.x; v[1] = x.y;
        }
    }
    __device__ __forceinline__ void zero()
    {
#pragma unroll
        for (int i = 0; i < kWords; ++i) v[i] = 0u;
    }
};

__device__ __forceinline__ void mma_e4m3_16832(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Query side of the scan for one row t: the B fragments of q^I_t (heads as
// MMA columns, d in the same byte permutation as KeyQuarter) and the head
// weights w_t, in the lanes that use them.
template <int NT, int DI>
struct QueryFrag {
    static constexpr int KSTEPS = DI / 32;
    uint32_t bq[NT][KSTEPS][2];
    float wv[NT][2];

    __device__ __forceinline__ void load(const uint8_t* __restrict__ q_idx, const float* __restrict__ w,
                                         int t, int H_I, int lane)
    {
        const int gid = lane >> 2, tid4 = lane & 3;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int h = nt * 8 + gid;
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
                if (h < H_I) {
                    const uint2 x = *reinterpret_cast<const uint2*>(
                        q_idx + ((size_t)t * H_I + h) * DI + tid4 * (DI / 4) + 8 * kk);
                    bq[nt][kk][0] = x.x;
                    bq[nt][kk][1] = x.y;
                } else {
                    bq[nt][kk][0] = bq[nt][kk][1] = 0u;
                }
            }
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int h2 = nt * 8 + 2 * tid4 + e;
                wv[nt][e] = h2 < H_I ? w[(size_t)t * H_I + h2] : 0.f;
            }
        }
    }

    // I for key rows A (MMA rows 0-7) and B (rows 8-15) of a 16-key block;
    // the full sums end up in every lane (reduced over the quad).
    __device__ __forceinline__ void score(const KeyQuarter<DI>& A, const KeyQuarter<DI>& B,
                                          float& ia, float& ib) const
    {
        ia = 0.f;
        ib = 0.f;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk)
                mma_e4m3_16832(acc, A.v[2 * kk], B.v[2 * kk], A.v[2 * kk + 1], B.v[2 * kk + 1],
                               bq[nt][kk][0], bq[nt][kk][1]);
            ia = fmaf(wv[nt][0], fmaxf(acc[0], 0.f), ia);
            ia = fmaf(wv[nt][1], fmaxf(acc[1], 0.f), ia);
            ib = fmaf(wv[nt][0], fmaxf(acc[2], 0.f), ib);
            ib = fmaf(wv[nt][1], fmaxf(acc[3], 0.f), ib);
        }
        ia += __shfl_xor_sync(0xffffffffu, ia, 1);
        ib += __shfl_xor_sync(0xffffffffu, ib, 1);
        ia += __shfl_xor_sync(0xffffffffu, ia, 2);
        ib += __shfl_xor_sync(0xffffffffu, ib, 2);
    }
};

constexpr int kScoreThreads = 128;

// Grid: x = key block (keys_per_cta keys), y = query row r (t = row0 + r).
// scores[r * ld + s] = I_{t,s} for s in the block and s <= pos[t].
template <int NT, int DI>
__global__ void __launch_bounds__(kScoreThreads)
indexer_scores_kernel(const uint8_t* __restrict__ q_idx, const float* __restrict__ w,
                      const uint8_t* __restrict__ k_idx, const int* __restrict__ pos,
                      const int* __restrict__ k_base, int T, int S, int H_I, int row0,
                      float* __restrict__ scores, long long ld, int keys_per_cta)
{
    const int r = blockIdx.y;
    const int t = row0 + r;
    long long base;
    const int n = row_candidates(pos, k_base, t, T, S, &base);
    const int s_begin = blockIdx.x * keys_per_cta;
    if (s_begin >= n) return;
    const int s_end = min(n, s_begin + keys_per_cta);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tid4 = lane & 3;
    QueryFrag<NT, DI> qf;
    qf.load(q_idx, w, t, H_I, lane);

    float* out = scores + (size_t)r * ld;
    constexpr int kWarps = kScoreThreads / 32;
    for (int s0 = s_begin + warp * 16; s0 < s_end; s0 += kWarps * 16) {
        const int sa = s0 + gid, sb = s0 + gid + 8;
        KeyQuarter<DI> A, B;
        if (sa < s_end) A.load(k_idx + (size_t)(base + sa) * DI + tid4 * (DI / 4)); else A.zero();
        if (sb < s_end) B.load(k_idx + (size_t)(base + sb) * DI + tid4 * (DI / 4)); else B.zero();
        float ia, ib;
        qf.score(A, B, ia, ib);
        if (tid4 == 0) {
            if (sa < s_end) out[sa] = ia;
            if (sb < s_end) out[sb] = ib;
        }
    }
}

}  // namespace dsa
