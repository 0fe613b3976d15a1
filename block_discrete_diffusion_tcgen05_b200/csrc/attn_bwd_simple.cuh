// attn_bwd_simple.cuh -- backward of the E2D2 train calls (encoder block-causal self-attention
// and the decoder's fused self+cross attention over 2L keys; "Encoder-Decoder Diffusion Language
// Models for Efficient Training and Inference", paper notes, sec. 4: one encoder and one decoder
// pass with custom masks train all blocks; the page gives no backward, so this is the plain
// derivative of those two attention calls that a gradient step through them needs).
//
// First, plain version on the CUDA cores (fp32 arithmetic, bf16 in and out), recomputing the
// probabilities from the forward's LSE:
//     p_ij  = exp(scale q_i.k_j - lse_i)            over the keys row i attends
//     dp_ij = dout_i . v_j
//     D_i   = sum_j p_ij dp_ij                      (= dout_i . out_i in exact arithmetic)
//     ds_ij = p_ij (dp_ij - D_i)
//     dq_i  = scale (sum_j p_ij dp_ij k_j - D_i sum_j p_ij k_j)
//                                                   (kernel 1, one warp per query row, one pass)
//     dv_j  = sum_i p_ij dout_i,  dk_j = scale sum_i ds_ij q_i
//                                                   (kernel 2, one warp per key row, over the
//                                                    query heads sharing the kv head)
// D_i is formed from the probabilities, not from the forward's bf16 output: where one key holds
// nearly all of a row's weight, dp_ij - D_i cancels, and out's bf16 rounding (relative 2^-9 per
// element, summed over the head dim) would then dominate ds_ij.
// A warp spreads the head dim over its lanes (D/32 values per lane) and reduces dot products with
// shuffles.  The key set of a query row / the query set of a key row are index ranges:
//     encoder     row i: keys [0, min(L, (blk(i)+1) S));   key j: queries [blk(j) S, L)
//     decoder     row i: encoder-side keys [0, blk(i) S), decoder-side keys [blk(i) S, min(L, (blk(i)+1) S))
//                 encoder-side key j: queries [(blk(j)+1) S, L); decoder-side key j: queries
//                 [blk(j) S, min(L, (blk(j)+1) S))
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace e2d2 {

struct BwdParams {
    const __nv_bfloat16* q;      // [B][Hq][L][D]
    const __nv_bfloat16* k0;     // encoder: k; decoder: k_enc       [B][Hkv][L][D]
    const __nv_bfloat16* v0;
    const __nv_bfloat16* k1;     // decoder: k_dec (null for the encoder)
    const __nv_bfloat16* v1;
    const float* lse;            // forward LSE [B][Hq][L] (natural log)
    const __nv_bfloat16* dout;   // [B][Hq][L][D]
    __nv_bfloat16* dq;           // [B][Hq][L][D]
    __nv_bfloat16* dk0;          // [B][Hkv][L][D]
    __nv_bfloat16* dv0;
    __nv_bfloat16* dk1;          // decoder only
    __nv_bfloat16* dv1;
    float* dsum;                 // workspace: D_i [B][Hq][L]
    int batch, q_heads, kv_heads, group, L, S;
    float scale;                 // natural-log units
    int decoder;
};

template <int D>
__device__ __forceinline__ void load_row(const __nv_bfloat16* row, int lane, float (&x)[D / 32]) {
#pragma unroll
    for (int e = 0; e < D / 32; ++e) x[e] = __bfloat162float(row[lane * (D / 32) + e]);
}

template <int D>
__device__ __forceinline__ float warp_dot(const float (&a)[D / 32], const float (&b)[D / 32]) {
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < D / 32; ++e) s = fmaf(a[e], b[e], s);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}

// Kernel 1: dq and D_i, one warp per query row (grid-stride over the B*Hq*L rows).  Kernel 2
// reads D_i from `dsum`, so it runs after this one on the same stream.
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_dq_kernel(const BwdParams p) {
    constexpr int E = D / 32;
    const int lane = threadIdx.x % 32;
    const long long rows = static_cast<long long>(p.batch) * p.q_heads * p.L;
    const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
    for (long long r = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32; r < rows; r += warps) {
        const int i = static_cast<int>(r % p.L);
        const long long bh = r / p.L;
        const int h = static_cast<int>(bh % p.q_heads);
        const int b = static_cast<int>(bh / p.q_heads);
        const long long kvz = static_cast<long long>(b) * p.kv_heads + h / p.group;
        float qi[E], gi[E], acc_pdk[E], acc_pk[E];
        load_row<D>(p.q + r * D, lane, qi);
        load_row<D>(p.dout + r * D, lane, gi);
        const float lse = p.lse[r];
        float Di = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) acc_pdk[e] = acc_pk[e] = 0.f;
        const int b0 = (i / p.S) * p.S;
        const int bend = min(p.L, b0 + p.S);
        // encoder: keys [0, bend) of k0/v0.  decoder: keys [0, b0) of k0/v0, then [b0, bend) of k1/v1.
        for (int src = 0; src < (p.decoder ? 2 : 1); ++src) {
            const __nv_bfloat16* K = (src == 0 ? p.k0 : p.k1) + kvz * p.L * D;
            const __nv_bfloat16* V = (src == 0 ? p.v0 : p.v1) + kvz * p.L * D;
            const int j0 = (p.decoder && src == 1) ? b0 : 0;
            const int j1 = p.decoder ? (src == 0 ? b0 : bend) : bend;
            for (int j = j0; j < j1; ++j) {
                float kj[E], vj[E];
                load_row<D>(K + static_cast<long long>(j) * D, lane, kj);
                load_row<D>(V + static_cast<long long>(j) * D, lane, vj);
                const float pij = expf(p.scale * warp_dot<D>(qi, kj) - lse);
                const float pdp = pij * warp_dot<D>(gi, vj);
                Di += pdp;
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    acc_pdk[e] = fmaf(pdp, kj[e], acc_pdk[e]);
                    acc_pk[e] = fmaf(pij, kj[e], acc_pk[e]);
                }
            }
        }
#pragma unroll
        for (int e = 0; e < E; ++e)
            p.dq[r * D + lane * E + e] = __float2bfloat16_rn(p.scale * fmaf(-Di, acc_pk[e], acc_pdk[e]));
        if (lane == 0) p.dsum[r] = Di;
    }
}

// Kernel 2: dk and dv, one warp per key row of each source (grid-stride over B*Hkv*L*sources).
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_dkv_kernel(const BwdParams p) {
    constexpr int E = D / 32;
    const int lane = threadIdx.x % 32;
    const int nsrc = p.decoder ? 2 : 1;
    const long long keys = static_cast<long long>(p.batch) * p.kv_heads * p.L;
    const long long total = keys * nsrc;
    const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
    for (long long w = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32; w < total; w += warps) {
        const int src = static_cast<int>(w / keys);
        const long long kr = w % keys;  // (b*Hkv + g)*L + j
        const int j = static_cast<int>(kr % p.L);
        const long long kvz = kr / p.L;
        const int g = static_cast<int>(kvz % p.kv_heads);
        const int b = static_cast<int>(kvz / p.kv_heads);
        float kj[E], vj[E], dk[E], dv[E];
        load_row<D>((src == 0 ? p.k0 : p.k1) + kr * D, lane, kj);
        load_row<D>((src == 0 ? p.v0 : p.v1) + kr * D, lane, vj);
#pragma unroll
        for (int e = 0; e < E; ++e) dk[e] = dv[e] = 0.f;
        const int bj = (j / p.S) * p.S;
        int i0, i1;
        if (!p.decoder) {
            i0 = bj;
            i1 = p.L;
        } else if (src == 0) {
            i0 = min(p.L, bj + p.S);  // queries of later blocks
            i1 = p.L;
        } else {
            i0 = bj;                  // queries of the same block
            i1 = min(p.L, bj + p.S);
        }
        for (int h = g * p.group; h < (g + 1) * p.group; ++h) {
            const long long rbase = (static_cast<long long>(b) * p.q_heads + h) * p.L;
            for (int i = i0; i < i1; ++i) {
                const long long r = rbase + i;
                float qi[E], gi[E];
                load_row<D>(p.q + r * D, lane, qi);
                load_row<D>(p.dout + r * D, lane, gi);
                const float pij = expf(p.scale * warp_dot<D>(qi, kj) - p.lse[r]);
                const float ds = pij * (warp_dot<D>(gi, vj) - p.dsum[r]);
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    dv[e] = fmaf(pij, gi[e], dv[e]);
                    dk[e] = fmaf(ds, qi[e], dk[e]);
                }
            }
        }
        __nv_bfloat16* DK = (src == 0 ? p.dk0 : p.dk1) + kr * D;
        __nv_bfloat16* DV = (src == 0 ? p.dv0 : p.dv1) + kr * D;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            DK[lane * E + e] = __float2bfloat16_rn(p.scale * dk[e]);
            DV[lane * E + e] = __float2bfloat16_rn(dv[e]);
        }
    }
}

}  // namespace e2d2
