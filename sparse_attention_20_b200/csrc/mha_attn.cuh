// MLA in MHA mode: causal attention in which every head has its own key and
// value rows (the latent row expanded per head), as opposed to the MQA mode of
// the sparse path where one latent row serves all heads (the bilingual paper
// summary's section list, "Appendix A MHA and MQA Modes of MLA"; "Paper
// Breakdown: DeepSeek-V3.2", section 2, "DSA under MLA (MQA Mode)"). For a
// short prefill (L <= k) the selector keeps every causal key, so the mode is
// dense causal attention:
//   o_{t,h} = sum_{s <= pos[t]} softmax_s(scale q_{t,h}.k_{s,h}) v_{s,h},
//   lse_{t,h} = log sum_{s <= pos[t]} exp(scale q_{t,h}.k_{s,h}),  pos[t] = t + S - T.
//
// One CTA per (128 query rows, head), 8 warps of 16 rows. The warp keeps its
// query fragments in registers, streams 64-key tiles of K and V through
// double-buffered shared memory (cp.async), forms the logits with warp-level
// bf16 MMAs, keeps a running max and sum per row (online softmax, log2
// domain) and feeds the bf16 probabilities straight from the accumulator
// registers into the P.V MMAs.
#pragma once
#include "attn_bwd.cuh"
#include "common.cuh"
#include "sm100.cuh"

namespace dsa {
namespace mha {

using dsa::bwd::bk_addr;
using dsa::bwd::bn_addr;
using dsa::bwd::cp_async_commit;
using dsa::bwd::cp_async_wait_group;
using dsa::bwd::ldsm_x4;
using dsa::bwd::ldsm_x4_t;
using dsa::bwd::ld_pair;
using dsa::bwd::mma_bf16;
using sm100::smem_u32;

constexpr int kRows = 128;   // query rows per CTA
constexpr int kKeys = 64;    // keys per tile
constexpr int kThreads = 256;

template <int DH, int DV>
struct Shape {
    static_assert(DH % 16 == 0 && DV % 16 == 0, "head dims must be multiples of 16");
    static constexpr int LDK = DH + 8, LDV = DV + 8;   // padded rows: conflict-free ldmatrix
    static constexpr int kStage = kKeys * (LDK + LDV);
    static constexpr size_t kSmem = 2 * (size_t)kStage * sizeof(__nv_bfloat16);
};

// grid: x = query tile, y = head. q [T][Hq][DH], k [S][Hq][DH], v [S][Hq][DV] bf16;
// out [T][Hq][DV] bf16, lse [T][Hq] fp32. Requires T <= S.
template <int DH, int DV>
__global__ void __launch_bounds__(kThreads, 1)
mha_causal_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                  const __nv_bfloat16* __restrict__ v, int T, int S, int Hq, float scale,
                  __nv_bfloat16* __restrict__ out, float* __restrict__ lse)
{
    using Sh = Shape<DH, DV>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __nv_bfloat16* stage0 = reinterpret_cast<__nv_bfloat16*>(smem_raw);

    // the last query tiles see the most keys: launch them first so the short
    // tiles fill the tail of the grid
    const int t0 = (gridDim.x - 1 - blockIdx.x) * kRows, h = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, tq = lane & 3;
    const int rA = t0 + warp * 16 + gq, rB = rA + 8;
    const int shift = S - T;   // pos[t] = t + shift
    constexpr float kLog2e = 1.4426950408889634f;
    const float zs = scale * kLog2e;

    // keys the CTA and the warp need
    const int kmax = min(S, t0 + kRows + shift);
    const int wmax = min(S, t0 + warp * 16 + 16 + shift);
    const int n_tiles = (kmax + kKeys - 1) / kKeys;

    auto load_tile = [&](int it) {
        __nv_bfloat16* ks = stage0 + (size_t)(it & 1) * Sh::kStage;
        __nv_bfloat16* vs = ks + kKeys * Sh::LDK;
        const int s0 = it * kKeys;
        for (int e = threadIdx.x; e < kKeys * (DH / 8); e += kThreads) {
            const int j = e / (DH / 8), c8 = (e - j * (DH / 8)) * 8;
            const bool ok = s0 + j < S;
            const __nv_bfloat16* src = ok ? k + ((size_t)(s0 + j) * Hq + h) * DH + c8 : k;
            sm100::cp_async16(smem_u32(ks + j * Sh::LDK + c8), src, ok ? 16u : 0u);
        }
        for (int e = threadIdx.x; e < kKeys * (DV / 8); e += kThreads) {
            const int j = e / (DV / 8), c8 = (e - j * (DV / 8)) * 8;
            const bool ok = s0 + j < S;
            const __nv_bfloat16* src = ok ? v + ((size_t)(s0 + j) * Hq + h) * DV + c8 : v;
            sm100::cp_async16(smem_u32(vs + j * Sh::LDV + c8), src, ok ? 16u : 0u);
        }
        cp_async_commit();
    };
    if (n_tiles > 0) load_tile(0);

    // query fragments of rows rA, rB (zeros past T)
    uint32_t qa[DH / 16][4];
    {
        const bool okA = rA < T, okB = rB < T;
        const __nv_bfloat16* qA = q + ((size_t)(okA ? rA : 0) * Hq + h) * DH + 2 * tq;
        const __nv_bfloat16* qB = q + ((size_t)(okB ? rB : 0) * Hq + h) * DH + 2 * tq;
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
            qa[kk][0] = okA ? ld_pair(qA + kk * 16) : 0u;
            qa[kk][1] = okB ? ld_pair(qB + kk * 16) : 0u;
            qa[kk][2] = okA ? ld_pair(qA + kk * 16 + 8) : 0u;
            qa[kk][3] = okB ? ld_pair(qB + kk * 16 + 8) : 0u;
        }
    }
    float o[DV / 8][4];
#pragma unroll
    for (int n = 0; n < DV / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[n][e] = 0.f;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    const int posA = rA + shift, posB = rB + shift;

    for (int it = 0; it < n_tiles; ++it) {
        if (it + 1 < n_tiles) {
            load_tile(it + 1);
            cp_async_wait_group<1>();
        } else {
            cp_async_wait_group<0>();
        }
        __syncthreads();
        const int s0 = it * kKeys;
        if (s0 < wmax) {
            const uint32_t k_u = smem_u32(stage0 + (size_t)(it & 1) * Sh::kStage);
            const uint32_t v_u = k_u + 2u * kKeys * Sh::LDK;
            float sc[8][4];
#pragma unroll
            for (int n = 0; n < 8; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) sc[n][e] = 0.f;
#pragma unroll
            for (int kk = 0; kk < DH / 16; ++kk) {
                uint32_t b[4][4];
#pragma unroll
                for (int np = 0; np < 4; ++np) ldsm_x4(bn_addr(k_u, Sh::LDK, np * 16, kk * 16, lane), b[np]);
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    mma_bf16(sc[2 * np], qa[kk], b[np][0], b[np][1]);
                    mma_bf16(sc[2 * np + 1], qa[kk], b[np][2], b[np][3]);
                }
            }
            // causal mask, log2-domain logits, running max
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int n = 0; n < 8; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int s = s0 + n * 8 + 2 * tq + (e & 1);
                    const bool ok = s <= ((e & 2) ? posB : posA);
                    const float x = ok ? sc[n][e] * zs : -INFINITY;
                    sc[n][e] = x;
                    mx[e >> 1] = fmaxf(mx[e >> 1], x);
                }
            float alpha[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
                mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
                const float mn = fmaxf(m[r], mx[r]);
                alpha[r] = mn == -INFINITY ? 1.f : exp2f(m[r] - mn);
                m[r] = mn;
                l[r] *= alpha[r];
            }
#pragma unroll
            for (int n = 0; n < DV / 8; ++n) {
                o[n][0] *= alpha[0];
                o[n][1] *= alpha[0];
                o[n][2] *= alpha[1];
                o[n][3] *= alpha[1];
            }
            uint32_t pa[4][4];
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                float p[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float mr = m[e >> 1];
                    p[e] = mr == -INFINITY ? 0.f : exp2f(sc[n][e] - mr);
                    l[e >> 1] += p[e];
                }
                // accumulator tile n -> A fragment of keys 16 (n / 2) .. + 16
                pa[n >> 1][(n & 1) * 2] = pack_bf16x2(p[0], p[1]);
                pa[n >> 1][(n & 1) * 2 + 1] = pack_bf16x2(p[2], p[3]);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
                for (int np = 0; np < DV / 16; ++np) {
                    uint32_t b[4];
                    ldsm_x4_t(bk_addr(v_u, Sh::LDV, np * 16, kk * 16, lane), b);
                    mma_bf16(o[2 * np], pa[kk], b[0], b[1]);
                    mma_bf16(o[2 * np + 1], pa[kk], b[2], b[3]);
                }
            }
        }
        __syncthreads();
    }
    // finish the row sums across the quad, normalise, write
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
        l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
    }
    const float inv[2] = {l[0] > 0.f ? 1.f / l[0] : 0.f, l[1] > 0.f ? 1.f / l[1] : 0.f};
    constexpr float kLn2 = 0.6931471805599453f;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int row = r ? rB : rA;
        if (row >= T) continue;
        __nv_bfloat16* dst = out + ((size_t)row * Hq + h) * DV + 2 * tq;
#pragma unroll
        for (int n = 0; n < DV / 8; ++n)
            *reinterpret_cast<uint32_t*>(dst + n * 8) =
                pack_bf16x2(o[n][2 * r] * inv[r], o[n][2 * r + 1] * inv[r]);
        if (tq == 0) lse[(size_t)row * Hq + h] = l[r] > 0.f ? (m[r] + __log2f(l[r])) * kLn2 : -INFINITY;
    }
}

}  // namespace mha
}  // namespace dsa
