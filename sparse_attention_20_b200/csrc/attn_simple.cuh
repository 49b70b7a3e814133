// Sparse MQA attention on CUDA cores, for any (Hq, d_qk, d_v) in the supported
// set: the general path for shapes the tensor-core kernel does not take, and
// the split + log-sum-exp merge used when few query rows must fill the GPU.
//
//   u_t = Attn(h_t, {c_s : s selected}); MLA in MQA mode, one latent row c_s
//   shared by every head ("Paper Breakdown: DeepSeek-V3.2", section 2,
//   "Attention" and "DSA under MLA (MQA Mode)").
//
// One CTA handles one query row, 8 heads and one split (a contiguous part of
// the row's selected entries). Logits stay in shared memory; the value pass
// streams each selected row once, coalesced, for all 8 heads.
#pragma once
#include "common.cuh"

namespace dsa {

constexpr int kAttnHeads = 8;
constexpr int kAttnThreads = 256;

__host__ __device__ inline size_t attn_simple_smem(int d_qk, int kcap)
{
    return sizeof(float) * ((size_t)kAttnHeads * d_qk + (size_t)kAttnHeads * kcap) +
           sizeof(int) * ((size_t)kcap + 64);
}

// grid: x = query row t, y = head group (8 heads), z = split.
// splits == 1: writes out (bf16) and lse. Otherwise writes the split's
// normalised partial output and its lse to part_o [T, splits, Hq, d_v] and
// part_lse [T, splits, Hq].
__global__ void __launch_bounds__(kAttnThreads)
sparse_attn_simple_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kv,
                          const int* __restrict__ idx, const int* __restrict__ pos,
                          const int* __restrict__ k_base, int T, int S, int Hq, int d_qk, int d_v,
                          int k, int kcap, float scale, __nv_bfloat16* __restrict__ out,
                          float* __restrict__ lse, float* __restrict__ part_o,
                          float* __restrict__ part_lse)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float* qs = reinterpret_cast<float*>(smem_raw);          // [8][d_qk]
    float* logit = qs + kAttnHeads * d_qk;                     // [8][kcap]
    int* sel = reinterpret_cast<int*>(logit + kAttnHeads * kcap);  // [kcap]
    int* misc = sel + kcap;                                    // [64]
    float* mrow = reinterpret_cast<float*>(misc + 16);         // [8]
    float* lrow = mrow + kAttnHeads;                           // [8]

    const int t = blockIdx.x;
    const int h0 = blockIdx.y * kAttnHeads;
    const int split = blockIdx.z, splits = gridDim.z;
    const int nh = min(kAttnHeads, Hq - h0);
    long long base;
    const int n_cand = row_candidates(pos, k_base, t, T, S, &base);
    const int p = n_cand - 1;   // last valid s
    const int n_row = min(k, n_cand);
    const int per = ceil_div(n_row, splits);
    const int i0 = min(n_row, split * per), i1 = min(n_row, i0 + per);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // query heads -> fp32 in shared memory
    for (int e = threadIdx.x; e < kAttnHeads * d_qk; e += kAttnThreads) {
        const int h = e / d_qk, d = e - h * d_qk;
        qs[e] = h < nh ? __bfloat162float(q[((size_t)t * Hq + h0 + h) * d_qk + d]) : 0.f;
    }
    // ordered compaction of the valid entries of [i0, i1)
    if (threadIdx.x == 0) misc[0] = 0;
    __syncthreads();
    for (int c0 = i0; c0 < i1; c0 += kAttnThreads) {
        const int i = c0 + threadIdx.x;
        int s = -1;
        if (i < i1) s = idx[(size_t)t * k + i];
        const bool ok = (i < i1) && s >= 0 && s <= p;
        const unsigned m = __ballot_sync(0xffffffffu, ok);
        if (lane == 0) misc[32 + warp] = __popc(m);
        __syncthreads();
        int off = misc[0];
        for (int w = 0; w < warp; ++w) off += misc[32 + w];
        if (ok) sel[off + __popc(m & ((1u << lane) - 1u))] = s;
        __syncthreads();
        if (threadIdx.x == 0) {
            int tot = 0;
            for (int w = 0; w < kAttnThreads / 32; ++w) tot += misc[32 + w];
            misc[0] += tot;
        }
        __syncthreads();
    }
    const int nsel = misc[0];

    // logits: one selected row per thread, all 8 heads
    for (int i = threadIdx.x; i < nsel; i += kAttnThreads) {
        const uint4* row = reinterpret_cast<const uint4*>(kv + (size_t)(base + sel[i]) * d_qk);
        float dot[kAttnHeads];
#pragma unroll
        for (int h = 0; h < kAttnHeads; ++h) dot[h] = 0.f;
        for (int d8 = 0; d8 < d_qk / 8; ++d8) {
            const uint4 x = __ldg(row + d8);
            const float v[8] = {bf16_lo(x.x), bf16_hi(x.x), bf16_lo(x.y), bf16_hi(x.y),
                                bf16_lo(x.z), bf16_hi(x.z), bf16_lo(x.w), bf16_hi(x.w)};
#pragma unroll
            for (int h = 0; h < kAttnHeads; ++h) {
                const float* qh = qs + h * d_qk + d8 * 8;
#pragma unroll
                for (int e = 0; e < 8; ++e) dot[h] = fmaf(qh[e], v[e], dot[h]);
            }
        }
#pragma unroll
        for (int h = 0; h < kAttnHeads; ++h) logit[h * kcap + i] = dot[h] * scale;
    }
    __syncthreads();

    // softmax statistics, one warp per head; logits become exp(z - m)
    if (warp < kAttnHeads) {
        float* z = logit + warp * kcap;
        float m = -INFINITY;
        for (int i = lane; i < nsel; i += 32) m = fmaxf(m, z[i]);
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f;
        for (int i = lane; i < nsel; i += 32) {
            const float e = expf(z[i] - m);
            z[i] = e;
            l += e;
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (lane == 0) {
            mrow[warp] = m;
            lrow[warp] = l;
        }
    }
    __syncthreads();

    // values: thread owns column pairs, streams the selected rows once
    for (int c2 = threadIdx.x; c2 < d_v / 2; c2 += kAttnThreads) {
        float acc[kAttnHeads][2];
#pragma unroll
        for (int h = 0; h < kAttnHeads; ++h) acc[h][0] = acc[h][1] = 0.f;
        for (int i = 0; i < nsel; ++i) {
            const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(
                kv + (size_t)(base + sel[i]) * d_qk + 2 * c2));
            const float v0 = bf16_lo(v), v1 = bf16_hi(v);
#pragma unroll
            for (int h = 0; h < kAttnHeads; ++h) {
                const float pw = logit[h * kcap + i];
                acc[h][0] = fmaf(pw, v0, acc[h][0]);
                acc[h][1] = fmaf(pw, v1, acc[h][1]);
            }
        }
        for (int h = 0; h < nh; ++h) {
            const float l = lrow[h];
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const float o0 = acc[h][0] * inv, o1 = acc[h][1] * inv;
            if (splits == 1) {
                *reinterpret_cast<uint32_t*>(out + ((size_t)t * Hq + h0 + h) * d_v + 2 * c2) =
                    pack_bf16x2(o0, o1);
            } else {
                float* po = part_o + (((size_t)t * splits + split) * Hq + h0 + h) * d_v + 2 * c2;
                po[0] = o0;
                po[1] = o1;
            }
        }
    }
    if (threadIdx.x < nh) {
        const int h = threadIdx.x;
        const float l = lrow[h];
        const float v = l > 0.f ? mrow[h] + logf(l) : -INFINITY;
        if (splits == 1) lse[(size_t)t * Hq + h0 + h] = v;
        else part_lse[((size_t)t * splits + split) * Hq + h0 + h] = v;
    }
}

// Log-sum-exp merge of the splits of one (row, head): grid x = row, y = head.
__global__ void lse_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                                   int T, int Hq, int d_v, int splits, __nv_bfloat16* __restrict__ out,
                                   float* __restrict__ lse)
{
    const int t = blockIdx.x, h = blockIdx.y;
    float m = -INFINITY;
    for (int z = 0; z < splits; ++z) m = fmaxf(m, part_lse[((size_t)t * splits + z) * Hq + h]);
    float total = -INFINITY;
    if (m != -INFINITY) {
        float l = 0.f;
        for (int z = 0; z < splits; ++z) l += expf(part_lse[((size_t)t * splits + z) * Hq + h] - m);
        total = m + logf(l);
    }
    for (int c = threadIdx.x; c < d_v; c += blockDim.x) {
        float acc = 0.f;
        if (total != -INFINITY)
            for (int z = 0; z < splits; ++z) {
                const float lz = part_lse[((size_t)t * splits + z) * Hq + h];
                if (lz == -INFINITY) continue;
                acc = fmaf(expf(lz - total), part_o[(((size_t)t * splits + z) * Hq + h) * d_v + c],
                           acc);
            }
        out[((size_t)t * Hq + h) * d_v + c] = __float2bfloat16(acc);
    }
    if (threadIdx.x == 0) lse[(size_t)t * Hq + h] = total;
}

}  // namespace dsa
