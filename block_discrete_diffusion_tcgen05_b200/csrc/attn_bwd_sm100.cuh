// attn_bwd_sm100.cuh -- backward of the two E2D2 train calls on the B200 tensor cores (sm_100a):
// the encoder's block-causal self-attention and the decoder's fused self+cross attention over 2L
// keys ("Encoder-Decoder Diffusion Language Models for Efficient Training and Inference", paper
// notes, sec. 4: one encoder and one decoder pass with custom masks train all blocks).  The page
// prints no backward; this is the plain derivative of those two calls.
//
// With p_ij = exp(scale q_i.k_j - lse_i) over the pairs the forward's mask allows,
//     dp_ij = dout_i.v_j,   D_i = sum_j p_ij dp_ij,   ds_ij = p_ij (dp_ij - D_i),
//     dq_i = scale sum_j ds_ij k_j,   dk_j = scale sum_i ds_ij q_i,   dv_j = sum_i p_ij dout_i.
// Two launches of one warp-specialised template, deterministic (no atomics; every gradient
// element is written once by the CTA that owns its row):
//
//   kBwdRowsQ   one item = 128 query rows of one head (rows on the TMEM lanes); the keys the
//               rows see stream past in 64-key sub-tiles.  Per sub-tile
//                   S  = Q K^T,  dP = dO V^T                        (tcgen05.mma -> TMEM)
//                   p  = exp2(S scale log2e - lse_i log2e),  u = p (dp - c_i)
//                   Y += p K,    X += u K                          (A = p / u from TMEM)
//               with c_i = dout_i.out_i (out = the forward's output).  At the end
//                   D_i = c_i + sum_j u_ij,   dq_i = scale (X_i - (D_i - c_i) Y_i),
//               which is the formula above for ANY constant c_i (sum_j p_ij (dp_ij - D_i) k_j =
//               sum_j p_ij (dp_ij - c_i) k_j - (D_i - c_i) sum_j p_ij k_j); c_i close to D_i keeps
//               the bf16 operands u small where one key holds a row's weight, so the difference
//               X - (D - c) Y does not cancel to rounding noise.  -D_i and -lse_i log2e go to the
//               workspace for the second launch.
//   kBwdRowsKV  one item = 128 keys of one kv head and key source (keys on the TMEM lanes); the
//               queries of every head of the GQA group that see them stream past in 64-query
//               sub-tiles.  Per sub-tile
//                   S^T = K Q^T,  dP^T = V dO^T,  p^T = exp2(...),  ds^T = p^T (dp^T - D)
//                   dV += p^T dO,  dK += ds^T Q                      (A = p^T / ds^T from TMEM)
//               and the item writes dk = scale dK and dv = dV.
//
// The mask is per TMEM lane an interval of the column index (the keys a query row sees, or the
// queries that see a key), so sub-tiles outside every lane's interval are never loaded and no
// mask matrix exists.  Rows past L come in as zeros (TMA out-of-bounds fill) and their interval
// is empty; queries past L also carry lse = +inf in the workspace (p = 0).
//
// CTA = 12 warps: warp 0 issues the TMA loads (row tiles once per item, column sub-tiles through
// a ring), warp 1 owns tensor memory and issues the S / dP products, warp 2 issues the
// accumulations (two issuing threads, so neither stream waits behind the other), warp 3 fetches
// the per-row constants of the next item (rows-Q), warps 4..7 and 8..11 are two softmax
// warpgroups that take alternate sub-tiles and write the gradient tiles (through shared memory
// and one TMA store per tile, so the accumulator is free again at once).  Tensor memory holds three
// (S, dP) sets of 64 + 64 columns (two at head_dim 128), used round robin: while the warpgroups
// turn two sets into (p, u) the tensor core computes the products of the third and the
// accumulations of the sets already done, so a warpgroup normally finds its next S ready.  The two
// accumulators (Y, X or dV, dK) take the remaining 2 x head_dim columns.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "fmha_sm100.cuh"
#include "ptx_sm100.cuh"

namespace e2d2 {

enum BwdSide : int { kBwdRowsQ = 0, kBwdRowsKV = 1 };

constexpr int kBwdRows = 128;  // rows of an item (TMEM lanes)
constexpr int kBwdCols = 64;   // columns of a sub-tile
constexpr float kLog2e = 1.4426950408889634f;

struct alignas(64) BwdTcParams {
    CUtensorMap tm_ga[2];  // gradient stores (128-row boxes): rows-Q: dq at [0]; rows-KV: dv of key source 0/1
    CUtensorMap tm_gb[2];  // rows-KV: dk of key source 0/1
    CUtensorMap tm_r1[2];  // row operand 1 (128-row boxes): rows-Q: Q at [0]; rows-KV: K of key source 0/1
    CUtensorMap tm_r2[2];  // row operand 2: rows-Q: dO at [0]; rows-KV: V of key source 0/1
    CUtensorMap tm_c1[2];  // column operand 1 (64-row boxes): rows-Q: K of key source 0/1; rows-KV: Q at [0]
    CUtensorMap tm_c2[2];  // column operand 2: rows-Q: V of key source 0/1; rows-KV: dO at [0]
    CUtensorMap tm_out;    // rows-Q: the forward's output (128-row boxes), for c_i
    const float* lse;                 // rows-Q: the forward's lse [B*Hq][L] (natural log)
    const __nv_bfloat16* out;         // rows-Q: the forward's output [B*Hq][L][D]
    const __nv_bfloat16* dout;        // rows-Q: [B*Hq][L][D]
    float* ws_nl2;                    // [B*Hq][Lpad]: -lse*log2(e), -inf past L (rows-Q writes it)
    float* ws_D;                      // [B*Hq][Lpad]: -D_i, 0 past L
    __nv_bfloat16* g_a[2];            // rows-Q: dq at [0]; rows-KV: dv of key source 0/1
    __nv_bfloat16* g_b[2];            // rows-KV: dk of key source 0/1
    unsigned int* err;                // device error word
    int batch, q_heads, kv_heads, group;
    int L, S, Lpad, decoder;
    float scale, scale_log2;
    int n_row_tiles;                  // ceil(L / 128)
    int num_items;
};

template <int D>
struct BwdCfg {
    static constexpr int RB = (D * 2 < 128) ? D * 2 : 128;   // bytes per smem row of one chunk
    static constexpr int NCH = D * 2 / RB;                   // column chunks per row
    static constexpr uint32_t SWZ = (RB == 128) ? 2u : 4u;   // 128-byte / 64-byte swizzle
    static constexpr int ROW_CHUNK = kBwdRows * RB;
    static constexpr int ROW_TILE = kBwdRows * D * 2;
    static constexpr int COL_CHUNK = kBwdCols * RB;
    static constexpr int COL_TILE = kBwdCols * D * 2;
    static constexpr int KSTEPS_PER_CHUNK = RB / 32;         // 16-element k steps per chunk
    static constexpr int RBUF = (D == 128) ? 1 : 2;          // row-tile buffers (items in flight)
    static constexpr int NST = (D == 128) ? 2 : (D == 64 ? 6 : 8);  // column stages
    // (S, dP) sets of 128 TMEM columns and accumulator sets of 2 D columns, within 512 columns.
    // A third set lets the products of sub-tile n+2 run while sub-tile n's p is still consumed.
    static constexpr int NSET = (D == 128) ? 2 : 3;
    static constexpr int NACC = (D == 32) ? 2 : 1;
    static_assert(NSET * 128 + NACC * 2 * D <= 512, "tensor memory budget");
};

template <int D>
struct BwdSmem {
    using C = BwdCfg<D>;
    static constexpr int OFF_R = 0;                                        // [RBUF][2] row tiles
    static constexpr int OFF_C = OFF_R + C::RBUF * 2 * C::ROW_TILE;        // [NST][2] column tiles
    static constexpr int OFF_LD = OFF_C + C::NST * 2 * C::COL_TILE;        // [NST][2][64] nl2, -D
    static constexpr int OFF_X = OFF_LD + C::NST * 2 * kBwdCols * 4;       // [2][2][128] sum exchange
    static constexpr int OFF_ROWD = OFF_X + 2 * 2 * kBwdRows * 4;         // [2][2][128] rows-Q: c_i, -lse_i log2e
    static constexpr int OFF_STG = ((OFF_ROWD + 2 * 2 * kBwdRows * 4 + 1023) / 1024) * 1024;  // [2] gradient tiles
    // rows-Q stores one gradient tile: the second stage buffer holds the forward's out tile
    static constexpr int OFF_OUT = OFF_STG + C::ROW_TILE;
    static constexpr int OFF_BAR = OFF_STG + 2 * C::ROW_TILE;
    // row_full[RBUF], row_empty[RBUF], col_full[NST], col_empty[NST], s_full[NSET], p_full[NSET],
    // set_free[NSET], acc_full[NACC], acc_free[NACC], rowd_full[2], rowd_empty[2], out_full,
    // out_empty, acc_issued, mma_drain, acc_drain, softmax_done, usum_ready[2], stg_free
    static constexpr int NBAR = 2 * C::RBUF + 2 * C::NST + 3 * C::NSET + 2 * C::NACC + 4 + 3 + 3 + 3;
    static constexpr int OFF_MISC = ((OFF_BAR + NBAR * 8 + 15) / 16) * 16;
    static constexpr int BYTES = OFF_MISC + 64;
    static constexpr int ALLOC = ((BYTES + 1023) / 1024) * 1024 + 1024;  // + alignment slack
};

struct BwdItem {
    int row_z;    // z of the row tiles: rows-Q b*Hq+h; rows-KV b*Hkv+g
    int row0;     // first row (query or key index) of the item
    int src;      // rows-KV: key source of the item (decoder: 0 encoder-side, 1 decoder-side)
    int nsub;     // column sub-tiles
    int a1, n1;   // rows-Q: source-1 key sub-tiles [a1, a1+n1), visited first
    int n0;       // rows-Q: source-0 key sub-tiles [0, n0)
    int qa, nq;   // rows-KV: query sub-tiles [qa, qa+nq) of each head of the group
    int col_z0;   // rows-Q: b*Hkv + h/G; rows-KV: b*Hq + g*G (first query head of the group)
};

// Items in a fixed order that every role walks; longest first (static round robin over CTAs).
// Rounds of gridDim.x items go to the CTAs alternately forwards and backwards (boustrophedon), so
// the per-CTA sums of the decreasing item costs stay level.
template <int SIDE>
struct BwdScheduler {
    const BwdTcParams& p;
    int r;  // round
    __device__ explicit BwdScheduler(const BwdTcParams& prm) : p(prm), r(0) {}

    __device__ bool next(BwdItem& it) {
        const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
        const int k = r * G + ((r & 1) ? G - 1 - c : c);
        if (k >= p.num_items) return false;
        ++r;
        const int L = p.L, S = p.S;
        if (SIDE == kBwdRowsQ) {
            const int BH = p.batch * p.q_heads;
            const int qt = p.n_row_tiles - 1 - k / BH;  // later query tiles see more keys
            const int bh = k % BH;
            const int b = bh / p.q_heads, h = bh % p.q_heads;
            it.row_z = bh;
            it.row0 = qt * kBwdRows;
            it.src = 0;
            it.col_z0 = b * p.kv_heads + h / p.group;
            const int r_last = min(L, it.row0 + kBwdRows) - 1;
            const int blk0 = it.row0 / S, blkl = r_last / S;
            const int hi = min(L, (blkl + 1) * S);
            if (!p.decoder) {
                it.a1 = 0;
                it.n1 = 0;
                it.n0 = ceil_div_i(hi, kBwdCols);
            } else {
                it.a1 = (blk0 * S) / kBwdCols;
                it.n1 = ceil_div_i(hi, kBwdCols) - it.a1;
                it.n0 = ceil_div_i(blkl * S, kBwdCols);
            }
            it.nsub = it.n1 + it.n0;
            it.qa = it.nq = 0;
        } else {
            const int BH = p.batch * p.kv_heads;
            const int per_src = BH * p.n_row_tiles;
            const int src = k / per_src;  // decoder: encoder-side keys first (they see more queries)
            const int kk = k % per_src;
            const int kt = kk / BH, z = kk % BH;
            it.row_z = z;
            it.row0 = kt * kBwdRows;
            it.src = src;
            const int b = z / p.kv_heads, g = z % p.kv_heads;
            it.col_z0 = b * p.q_heads + g * p.group;
            const int k_last = min(L, it.row0 + kBwdRows) - 1;
            const int blk0 = it.row0 / S, blkl = k_last / S;
            int lo, hi;
            if (!p.decoder) {
                lo = blk0 * S;
                hi = L;
            } else if (src == 0) {
                lo = min(L, (blk0 + 1) * S);
                hi = L;
            } else {
                lo = blk0 * S;
                hi = min(L, (blkl + 1) * S);
            }
            it.qa = lo / kBwdCols;
            it.nq = (hi > lo) ? ceil_div_i(hi, kBwdCols) - it.qa : 0;
            it.nsub = it.nq * p.group;
            it.a1 = it.n1 = it.n0 = 0;
        }
        return true;
    }
};

// Column sub-tile t of an item: key source (rows-Q), first column (key or query index) and the
// z coordinate of its tensor map (and of the workspace row, rows-KV).
struct BwdCol {
    int src, y, z;
};

template <int SIDE>
__device__ __forceinline__ BwdCol bwd_col(const BwdItem& it, int t) {
    BwdCol r;
    if (SIDE == kBwdRowsQ) {
        if (t < it.n1) {
            r.src = 1;
            r.y = (it.a1 + t) * kBwdCols;
        } else {
            r.src = 0;
            r.y = (t - it.n1) * kBwdCols;
        }
        r.z = it.col_z0;
    } else {
        const int hh = t / it.nq;
        r.src = 0;
        r.y = (it.qa + t - hh * it.nq) * kBwdCols;
        r.z = it.col_z0 + hh;
    }
    return r;
}

// The allowed columns of this lane's row in source `src`: [lo, hi).
//   rows-Q (row = query i):  encoder keys [0, end(i)); decoder encoder-side keys [0, start(i)),
//                            decoder-side keys [start(i), end(i))
//   rows-KV (row = key j):   encoder queries [start(j), L); decoder encoder-side keys are seen by
//                            queries [end(j), L), decoder-side keys by [start(j), end(j))
// with start(x) = floor(x/S) S and end(x) = min(L, start(x) + S); an invalid row (>= L) sees nothing.
template <int SIDE>
__device__ __forceinline__ void bwd_interval(const BwdTcParams& p, int row, int src, int& lo, int& hi) {
    if (row >= p.L) {
        lo = 0;
        hi = 0;
        return;
    }
    const int start = (row / p.S) * p.S;
    const int end = min(p.L, start + p.S);
    if (SIDE == kBwdRowsQ) {
        if (!p.decoder) {
            lo = 0;
            hi = end;
        } else if (src == 0) {
            lo = 0;
            hi = start;
        } else {
            lo = start;
            hi = end;
        }
    } else {
        if (!p.decoder) {
            lo = start;
            hi = p.L;
        } else if (src == 0) {
            lo = end;
            hi = p.L;
        } else {
            lo = start;
            hi = end;
        }
    }
}

// One sub-tile of one warpgroup, one lane = one row: reads the 64 S and 64 dP columns of its set,
// writes p (bf16, packed over S columns 0..31) and u / ds (over dP columns 0..31), and returns
// sum(u) (rows-Q).  Columns outside [cmin, cmax) get p = 0.  The arithmetic runs on column pairs
// (packed fp32x2 FMA / add / multiply of sm_100), the exponentials one by one.
//   rows-Q:  exponent argument s*sl2 + nl2_row, u = p (dp - c_row)
//   rows-KV: exponent argument s*sl2 + nl2[c], ds = p (dp - D[c]); nl2 and -D of the sub-tile's 64
//            columns sit in shared memory at ld_saddr (64 floats, then 64 floats)
template <int SIDE>
__device__ __forceinline__ float bwd_subtile(uint32_t set_tmem, int cmin, int cmax, float sl2, float nl2_row,
                                             float c_row, uint32_t ld_saddr) {
    uint32_t sr[64], dr[64];
    ptx::tmem_ld32(set_tmem, sr);
    ptx::tmem_ld32(set_tmem + 32, sr + 32);
    ptx::tmem_ld32(set_tmem + 64, dr);
    ptx::tmem_ld32(set_tmem + 96, dr + 32);
    ptx::tmem_wait_ld();
    ptx::reg_fence<64>(sr);
    ptx::reg_fence<64>(dr);
    const float2 sl2v = make_float2(sl2, sl2);
    float2 usum = make_float2(0.f, 0.f);
#pragma unroll
    for (int a = 0; a < 2; ++a) {
        const bool mine = (cmin < 32 * a + 32) && (cmax > 32 * a);
        const bool live = __any_sync(0xffffffffu, mine);
        const bool whole = __all_sync(0xffffffffu, (cmin <= 32 * a) && (cmax >= 32 * a + 32));
        uint32_t pk[16], uk[16];
        if (live) {
#pragma unroll
            for (int c4 = 0; c4 < 32; c4 += 4) {
                const int col = 32 * a + c4;
                float2 nl[2], nd[2];
                if (SIDE == kBwdRowsKV) {
                    const float4 a4 = ptx::lds_f4(ld_saddr + col * 4);
                    const float4 b4 = ptx::lds_f4(ld_saddr + (kBwdCols + col) * 4);
                    nl[0] = make_float2(a4.x, a4.y);
                    nl[1] = make_float2(a4.z, a4.w);
                    nd[0] = make_float2(b4.x, b4.y);
                    nd[1] = make_float2(b4.z, b4.w);
                } else {
                    nl[0] = nl[1] = make_float2(nl2_row, nl2_row);
                    nd[0] = nd[1] = make_float2(-c_row, -c_row);
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int c = col + 2 * h;
                    const float2 sv = make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
                    const float2 dv = make_float2(__uint_as_float(dr[c]), __uint_as_float(dr[c + 1]));
                    const float2 x = __ffma2_rn(sv, sl2v, nl[h]);
                    float2 pv = make_float2(ptx::ex2(x.x), ptx::ex2(x.y));
                    if (!whole) {
                        pv.x = (c >= cmin && c < cmax) ? pv.x : 0.f;
                        pv.y = (c + 1 >= cmin && c + 1 < cmax) ? pv.y : 0.f;
                    }
                    const float2 uv = __fmul2_rn(pv, __fadd2_rn(dv, nd[h]));
                    if (SIDE == kBwdRowsQ) usum = __fadd2_rn(usum, uv);
                    pk[(c4 >> 1) + h] = ptx::pack_bf16x2(pv.x, pv.y);
                    uk[(c4 >> 1) + h] = ptx::pack_bf16x2(uv.x, uv.y);
                }
            }
        } else {
#pragma unroll
            for (int c = 0; c < 16; ++c) pk[c] = uk[c] = 0u;
        }
        ptx::tmem_st16(set_tmem + 16 * a, pk);
        ptx::tmem_st16(set_tmem + 64 + 16 * a, uk);
    }
    return usum.x + usum.y;
}

// Dot product of two bf16 rows of length D (16-byte loads), fp32.
template <int D>
__device__ __forceinline__ float row_dot_bf16(const __nv_bfloat16* a, const __nv_bfloat16* b) {
    const uint4* a4 = reinterpret_cast<const uint4*>(a);
    const uint4* b4 = reinterpret_cast<const uint4*>(b);
    float s[2] = {0.f, 0.f};
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
        const uint4 x = __ldg(a4 + i), y = __ldg(b4 + i);
        const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xs[j]));
            const float2 yf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ys[j]));
            s[j & 1] = fmaf(xf.x, yf.x, s[j & 1]);
            s[j & 1] = fmaf(xf.y, yf.y, s[j & 1]);
        }
    }
    return s[0] + s[1];
}

// Writes N columns of one gradient row: values * f, bf16, 16-byte stores.
template <int N>
__device__ __forceinline__ void store_row_bf16(__nv_bfloat16* dst, const float* v, float f) {
#pragma unroll
    for (int c = 0; c < N; c += 8) reinterpret_cast<uint4*>(dst)[c / 8] = pack8_bf16(v + c, f);
}

template <int D, int SIDE>
__global__ void __launch_bounds__(kThreads, 1) attn_bwd_sm100_kernel(const __grid_constant__ BwdTcParams p) {
    using C = BwdCfg<D>;
    using SM = BwdSmem<D>;
    constexpr int NST = C::NST, RBUF = C::RBUF, NACC = C::NACC, NSET = C::NSET;
    constexpr uint32_t ACC0 = NSET * 128;  // first accumulator column
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    ptx::griddep_launch_dependents();  // the next kernel may launch; it waits for this one's end
#define E2D2_BWD_SMEM_POINTERS                                                                       \
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &      \
                                               ~static_cast<uintptr_t>(1023));                       \
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::OFF_BAR);                                \
    uint64_t* row_full = bars;                                                                       \
    uint64_t* row_empty = row_full + RBUF;                                                           \
    uint64_t* col_full = row_empty + RBUF;                                                           \
    uint64_t* col_empty = col_full + NST;                                                            \
    uint64_t* s_full = col_empty + NST;                                                              \
    uint64_t* p_full = s_full + NSET;                                                                \
    uint64_t* set_free = p_full + NSET;                                                              \
    uint64_t* acc_full = set_free + NSET;                                                            \
    uint64_t* acc_free = acc_full + NACC;                                                            \
    uint64_t* rowd_full = acc_free + NACC;                                                           \
    uint64_t* rowd_empty = rowd_full + 2;                                                            \
    uint64_t* out_full = rowd_empty + 2;                                                             \
    uint64_t* out_empty = out_full + 1;                                                              \
    uint64_t* acc_issued = out_empty + 1;                                                            \
    uint64_t* mma_drain = acc_issued + 1;                                                            \
    uint64_t* acc_drain = mma_drain + 1;                                                             \
    uint64_t* softmax_done = acc_drain + 1;                                                          \
    uint64_t* usum_ready = softmax_done + 1; /* rows-Q: [2] the early warpgroup's sum of u is in */  \
    uint64_t* stg_free = usum_ready + 2;     /* rows-Q: the last gradient store has read the stage */\
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SM::OFF_MISC);                        \
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM::OFF_MISC + 8);             \
    (void)row_full; (void)row_empty; (void)col_full; (void)col_empty; (void)s_full; (void)p_full;    \
    (void)acc_full; (void)acc_free; (void)mma_drain; (void)softmax_done; (void)tmem_holder;          \
    (void)set_free; (void)acc_drain; (void)rowd_full; (void)rowd_empty; (void)out_full;              \
    (void)out_empty; (void)acc_issued; (void)usum_ready; (void)stg_free;                             \
    (void)abort_flag;
    uint32_t tmem_base;
    {
        E2D2_BWD_SMEM_POINTERS
        if (threadIdx.x == 0) {
            for (int i = 0; i < RBUF; ++i) {
                ptx::mbar_init(&row_full[i], 1);
                // rows-Q: warp 3 also reads the dO tile (for c_i) before the buffer is reused
                ptx::mbar_init(&row_empty[i], SIDE == kBwdRowsQ ? 2 : 1);
            }
            for (int i = 0; i < NST; ++i) {
                ptx::mbar_init(&col_full[i], 1);
                ptx::mbar_init(&col_empty[i], 1);
            }
            for (int i = 0; i < NSET; ++i) {
                ptx::mbar_init(&s_full[i], 1);
                ptx::mbar_init(&p_full[i], 128);
                ptx::mbar_init(&set_free[i], 1);
            }
            for (int i = 0; i < NACC; ++i) {
                ptx::mbar_init(&acc_full[i], 1);
                ptx::mbar_init(&acc_free[i], kSoftmaxThreads);
            }
            for (int i = 0; i < 2; ++i) {
                ptx::mbar_init(&rowd_full[i], 32);
                ptx::mbar_init(&rowd_empty[i], kSoftmaxThreads);
            }
            ptx::mbar_init(out_full, 1);
            ptx::mbar_init(out_empty, 1);
            ptx::mbar_init(acc_issued, 1);
            ptx::mbar_init(mma_drain, 1);
            ptx::mbar_init(acc_drain, 1);
            ptx::mbar_init(softmax_done, kSoftmaxThreads);
            ptx::mbar_init(&usum_ready[0], 128);
            ptx::mbar_init(&usum_ready[1], 128);
            ptx::mbar_init(stg_free, 1);
            *abort_flag = 0;
            ptx::fence_mbar_init();
        }
        if (warp == 1) {
            ptx::tmem_alloc(tmem_holder, kTmemCols);
            ptx::tmem_relinquish();
        }
        ptx::griddep_wait();  // inputs (and the workspace) after the previous kernel has finished
        ptx::tc_fence_before();
        __syncthreads();
        ptx::tc_fence_after();
        tmem_base = *tmem_holder;
    }

    E2D2_BWD_SMEM_POINTERS
    const uint32_t smem_base = ptx::smem_u32(smem);
    const uint32_t sR = smem_base + SM::OFF_R;
    const uint32_t sC = smem_base + SM::OFF_C;

    if (warp == 0) {
        ptx::setmaxnreg_dec<kRegsControl>();
        // ------------------------------------------------------------------ TMA producer
        const bool leader = ptx::elect_one();
        if (leader) {
            for (int i = 0; i < 2; ++i) {
                ptx::tma_prefetch_desc(&p.tm_r1[i]);
                ptx::tma_prefetch_desc(&p.tm_r2[i]);
                ptx::tma_prefetch_desc(&p.tm_c1[i]);
                ptx::tma_prefetch_desc(&p.tm_c2[i]);
            }
        }
        __syncwarp();
        test_producer_delay();
        BwdScheduler<SIDE> sched(p);
        BwdItem it;
        uint32_t n = 0, iw = 0;
        bool ok = true;
        while (ok && sched.next(it)) {
            if (it.nsub == 0) continue;
            const uint32_t rb = iw % RBUF;
            ok = wait_bar_warp(&row_empty[rb], ((iw / RBUF) & 1) ^ 1, abort_flag, p.err);
            if (!ok) break;
            // debug builds: the row tile starts inside the sequence and its head exists
            E2D2_DCHECK(it.row0 < p.L && it.row_z < p.batch * (SIDE == kBwdRowsQ ? p.q_heads : p.kv_heads), p.err);
            if (leader) {
                const int rs = (SIDE == kBwdRowsQ) ? 0 : it.src;
                ptx::mbar_arrive_expect_tx(&row_full[rb], 2 * C::ROW_TILE);
                for (int ch = 0; ch < C::NCH; ++ch) {
                    ptx::tma_load_3d(&p.tm_r1[rs], &row_full[rb],
                                     smem + SM::OFF_R + (rb * 2 + 0) * C::ROW_TILE + ch * C::ROW_CHUNK,
                                     ch * (C::RB / 2), it.row0, it.row_z);
                    ptx::tma_load_3d(&p.tm_r2[rs], &row_full[rb],
                                     smem + SM::OFF_R + (rb * 2 + 1) * C::ROW_TILE + ch * C::ROW_CHUNK,
                                     ch * (C::RB / 2), it.row0, it.row_z);
                }
            }
            __syncwarp();
            if (SIDE == kBwdRowsQ) {
                // the forward's out tile of the item's rows (one buffer; warp 3 frees it)
                ok = wait_bar_warp(out_empty, (iw & 1u) ^ 1u, abort_flag, p.err);
                if (!ok) break;
                if (leader) {
                    ptx::mbar_arrive_expect_tx(out_full, C::ROW_TILE);
                    for (int ch = 0; ch < C::NCH; ++ch)
                        ptx::tma_load_3d(&p.tm_out, out_full, smem + SM::OFF_OUT + ch * C::ROW_CHUNK, ch * (C::RB / 2),
                                         it.row0, it.row_z);
                }
                __syncwarp();
            }
            ++iw;
            for (int t = 0; t < it.nsub; ++t) {
                const uint32_t st = n % NST;
                ok = wait_bar_warp(&col_empty[st], ((n / NST) & 1) ^ 1, abort_flag, p.err);
                if (!ok) break;
                const BwdCol cr = bwd_col<SIDE>(it, t);
                E2D2_DCHECK(cr.y < p.L && cr.z < p.batch * (SIDE == kBwdRowsQ ? p.kv_heads : p.q_heads), p.err);
                if (leader) {
                    const uint32_t bytes = 2 * C::COL_TILE + (SIDE == kBwdRowsKV ? 2 * kBwdCols * 4 : 0);
                    ptx::mbar_arrive_expect_tx(&col_full[st], bytes);
                    for (int ch = 0; ch < C::NCH; ++ch) {
                        ptx::tma_load_3d(&p.tm_c1[cr.src], &col_full[st],
                                         smem + SM::OFF_C + (st * 2 + 0) * C::COL_TILE + ch * C::COL_CHUNK,
                                         ch * (C::RB / 2), cr.y, cr.z);
                        ptx::tma_load_3d(&p.tm_c2[cr.src], &col_full[st],
                                         smem + SM::OFF_C + (st * 2 + 1) * C::COL_TILE + ch * C::COL_CHUNK,
                                         ch * (C::RB / 2), cr.y, cr.z);
                    }
                    if (SIDE == kBwdRowsKV) {
                        const size_t off = static_cast<size_t>(cr.z) * p.Lpad + cr.y;
                        ptx::bulk_load_g2s(smem + SM::OFF_LD + st * 2 * kBwdCols * 4, p.ws_nl2 + off, kBwdCols * 4,
                                           &col_full[st]);
                        ptx::bulk_load_g2s(smem + SM::OFF_LD + st * 2 * kBwdCols * 4 + kBwdCols * 4, p.ws_D + off,
                                           kBwdCols * 4, &col_full[st]);
                    }
                }
                __syncwarp();
                ++n;
            }
        }
        // Never leave with copies in flight: wait for the last load of every buffer.
        volatile int no_abort = 0;
        for (uint32_t i = n > static_cast<uint32_t>(NST) ? n - NST : 0u; i < n; ++i)
            wait_bar_warp(&col_full[i % NST], (i / NST) & 1u, &no_abort, p.err, true);
        for (uint32_t i = iw > static_cast<uint32_t>(RBUF) ? iw - RBUF : 0u; i < iw; ++i)
            wait_bar_warp(&row_full[i % RBUF], (i / RBUF) & 1u, &no_abort, p.err, true);
        if (SIDE == kBwdRowsQ && iw > 0) wait_bar_warp(out_full, (iw - 1) & 1u, &no_abort, p.err, true);
    } else if (warp == 1) {
        ptx::setmaxnreg_dec<kRegsControl>();
        // ------------------------------------------------------------------ product issuer
        // S = R1 C1^T and dP = R2 C2^T of every sub-tile into its set, once the set's previous
        // accumulation (sub-tile n - NSET, issued by warp 2) has read it.  Also owns tensor memory.
        const bool leader = ptx::elect_one();
        const uint64_t kdesc = ptx::smem_desc(0, 16, 8 * C::RB, C::SWZ);  // K-major
        constexpr uint32_t idesc_s = ptx::idesc_bf16_f32(kBwdRows, kBwdCols, false);
        BwdScheduler<SIDE> sched(p);
        BwdItem it;
        uint32_t n = 0, iw = 0;
        bool ok = true;
        while (ok && sched.next(it)) {
            if (it.nsub == 0) continue;
            const uint32_t rb = iw % RBUF;
            ok = wait_bar_warp(&row_full[rb], (iw / RBUF) & 1u, abort_flag, p.err);
            if (!ok) break;
            // The previous item's last accumulation goes to the tensor core before this item's
            // products, so its epilogue is not held up behind them.
            if (iw > 0) {
                ok = wait_bar_warp(acc_issued, (iw - 1) & 1u, abort_flag, p.err);
                if (!ok) break;
            }
            const uint32_t r1 = sR + (rb * 2 + 0) * C::ROW_TILE;
            const uint32_t r2 = sR + (rb * 2 + 1) * C::ROW_TILE;
            for (int t = 0; t < it.nsub && ok; ++t, ++n) {
                const uint32_t st = n % NST, set = n % NSET;
                ok = wait_bar_warp(&col_full[st], (n / NST) & 1u, abort_flag, p.err) &&
                     wait_bar_warp(&set_free[set], ((n / NSET) & 1u) ^ 1u, abort_flag, p.err);
                if (!ok) break;
                ptx::tc_fence_after();
                if (leader) {
                    const uint32_t c1 = sC + (st * 2 + 0) * C::COL_TILE;
                    const uint32_t c2 = sC + (st * 2 + 1) * C::COL_TILE;
                    const uint32_t sset = tmem_base + set * 128;
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t ro = (ks / C::KSTEPS_PER_CHUNK) * C::ROW_CHUNK + (ks % C::KSTEPS_PER_CHUNK) * 32;
                        const uint32_t co = (ks / C::KSTEPS_PER_CHUNK) * C::COL_CHUNK + (ks % C::KSTEPS_PER_CHUNK) * 32;
                        ptx::mma_ss(sset, kdesc | ((r1 + ro) >> 4), kdesc | ((c1 + co) >> 4), idesc_s, ks > 0 ? 1u : 0u);
                        ptx::mma_ss(sset + 64, kdesc | ((r2 + ro) >> 4), kdesc | ((c2 + co) >> 4), idesc_s,
                                    ks > 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(&s_full[set]);
                    if (t == it.nsub - 1) ptx::mma_commit(&row_empty[rb]);
                }
                __syncwarp();
            }
            ++iw;
        }
        // Drain: this warp's and warp 2's MMAs have completed and every softmax thread is done with
        // tensor memory before it is released.
        if (leader) ptx::mma_commit(mma_drain);
        __syncwarp();
        volatile int no_abort = 0;
        wait_bar_warp(mma_drain, 0, &no_abort, p.err, true);
        wait_bar_warp(acc_drain, 0, &no_abort, p.err, true);
        wait_bar_warp(softmax_done, 0, &no_abort, p.err, true);
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, kTmemCols);
    } else if (warp == 2) {
        ptx::setmaxnreg_dec<kRegsControl>();
        // ------------------------------------------------------------------ accumulation issuer
        // Y += p C1, X += u C1 (rows-Q) or dV += p^T C2, dK += ds^T C1 (rows-KV) of every sub-tile,
        // in order, once its softmax has written p and u into the set; then the set and the column
        // stage are free.
        const bool leader = ptx::elect_one();
        const uint64_t mndesc = ptx::smem_desc(0, C::COL_CHUNK, 8 * C::RB, C::SWZ);  // MN-major
        constexpr uint32_t idesc_o = ptx::idesc_bf16_f32(kBwdRows, D, true);
        BwdScheduler<SIDE> sched(p);
        BwdItem it;
        uint32_t n = 0, iw = 0;
        bool ok = true;
        while (ok && sched.next(it)) {
            if (it.nsub == 0) continue;
            const uint32_t ab = iw % NACC;
            for (int t = 0; t < it.nsub && ok; ++t, ++n) {
                const uint32_t set = n % NSET, st = n % NST;
                ok = wait_bar_warp(&p_full[set], (n / NSET) & 1u, abort_flag, p.err) &&
                     (t != 0 || wait_bar_warp(&acc_free[ab], ((iw / NACC) & 1u) ^ 1u, abort_flag, p.err));
                if (!ok) break;
                ptx::tc_fence_after();
                if (leader) {
                    const uint32_t c1 = sC + (st * 2 + 0) * C::COL_TILE;
                    const uint32_t c2 = sC + (st * 2 + 1) * C::COL_TILE;
                    const uint32_t ba = (SIDE == kBwdRowsQ) ? c1 : c2;
                    const uint32_t acc = tmem_base + ACC0 + ab * 2 * D;
                    const uint32_t pset = tmem_base + set * 128;
#pragma unroll
                    for (int ks = 0; ks < kBwdCols / 16; ++ks) {
                        const uint32_t accum = (t == 0 && ks == 0) ? 0u : 1u;
                        ptx::mma_ts(acc, pset + 8 * ks, mndesc | ((ba + ks * 16 * C::RB) >> 4), idesc_o, accum);
                        ptx::mma_ts(acc + D, pset + 64 + 8 * ks, mndesc | ((c1 + ks * 16 * C::RB) >> 4), idesc_o,
                                    accum);
                    }
                    ptx::mma_commit(&col_empty[st]);
                    ptx::mma_commit(&set_free[set]);
                    if (t == it.nsub - 1) {
                        ptx::mma_commit(&acc_full[ab]);
                        ptx::mbar_arrive(acc_issued);
                    }
                }
                __syncwarp();
            }
            ++iw;
        }
        if (leader) ptx::mma_commit(acc_drain);  // the thread that issued this warp's MMAs
        __syncwarp();
    } else if (warp == 3) {
        ptx::setmaxnreg_dec<kRegsControl>();
        // ------------------------------------------------------------------ row data (rows-Q)
        // c_i = dout_i.out_i and -lse_i log2(e) of the next item's 128 query rows into shared
        // memory, ahead of the softmax warpgroups (their global-load latency is off the critical
        // path); double-buffered by item.
        if (SIDE == kBwdRowsQ) {
            float* rowd = reinterpret_cast<float*>(smem + SM::OFF_ROWD);
            BwdScheduler<SIDE> sched(p);
            BwdItem it;
            uint32_t iw = 0;
            constexpr int UNITS_PER_CHUNK = C::RB / 16;
            while (sched.next(it)) {
                if (it.nsub == 0) continue;
                const uint32_t par = iw & 1u, rb = iw % RBUF;
                // -lse log2(e) of this lane's four rows (global loads issued first)
                float nl[kBwdRows / 32];
#pragma unroll
                for (int j = 0; j < kBwdRows / 32; ++j) {
                    const int row = it.row0 + j * 32 + lane;
                    nl[j] = row < p.L ? -__ldg(p.lse + static_cast<size_t>(it.row_z) * p.L + row) * kLog2e : 0.f;
                }
                wait_bar_warp(&rowd_empty[par], ((iw >> 1) & 1u) ^ 1u, abort_flag, p.err);
                wait_bar_warp(&row_full[rb], (iw / RBUF) & 1u, abort_flag, p.err);
                wait_bar_warp(out_full, iw & 1u, abort_flag, p.err);
                const uint8_t* tdo = smem + SM::OFF_R + (rb * 2 + 1) * C::ROW_TILE;
                const uint8_t* tout = smem + SM::OFF_OUT;
#pragma unroll
                for (int j = 0; j < kBwdRows / 32; ++j) {
                    const int lr = j * 32 + lane;
                    float2 acc2 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int unit = 0; unit < D / 8; ++unit) {
                        const uint32_t off = (unit / UNITS_PER_CHUNK) * C::ROW_CHUNK +
                                             swz_offset<C::RB>(lr, unit % UNITS_PER_CHUNK);
                        const uint4 x = *reinterpret_cast<const uint4*>(tdo + off);
                        const uint4 y = *reinterpret_cast<const uint4*>(tout + off);
                        const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            acc2 = __ffma2_rn(__bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xs[e])),
                                              __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ys[e])),
                                              acc2);
                    }
                    // rows past L: zero tiles (out-of-bounds fill), so c = 0
                    rowd[(par * 2 + 0) * kBwdRows + lr] = acc2.x + acc2.y;
                    rowd[(par * 2 + 1) * kBwdRows + lr] = nl[j];
                }
                __syncwarp();
                if (lane == 0) {
                    ptx::mbar_arrive(out_empty);
                    ptx::mbar_arrive(&row_empty[rb]);
                }
                ptx::mbar_arrive(&rowd_full[par]);
                ++iw;
            }
        }
    } else {
        ptx::setmaxnreg_inc<kRegsSoftmax>();
        // ------------------------------------------------------------------ softmax warpgroups
        // Warpgroup w (warps 4+4w .. 7+4w) takes the sub-tiles n with n % 2 == w (tensor-memory
        // set w).  Every thread owns one row (its TMEM lane).  Waits never break these loops, so
        // every warp takes every named barrier even after a bounded wait gave up.
        const int w = (warp - 4) >> 2;
        const int quarter = warp & 3;
        const int lrow = quarter * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const float sl2 = p.scale_log2;
        float* xch = reinterpret_cast<float*>(smem + SM::OFF_X);  // [2][2][128]
        BwdScheduler<SIDE> sched(p);
        BwdItem it;
        uint32_t n = 0, iw = 0;
        while (sched.next(it)) {
            const int row = it.row0 + lrow;
            const bool valid = row < p.L;
            if (it.nsub == 0) {
                // rows-KV only (every query row sees a key): keys that no query sees get zero
                // gradients.
                if (SIDE == kBwdRowsKV && valid) {
                    const float zero[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    __nv_bfloat16* dst = (w == 0 ? p.g_a[it.src] : p.g_b[it.src]) +
                                         (static_cast<size_t>(it.row_z) * p.L + row) * D;
#pragma unroll
                    for (int c = 0; c < D; c += 8) store_row_bf16<8>(dst + c, zero, 1.f);
                }
                continue;
            }
            int lo0, hi0, lo1, hi1;
            bwd_interval<SIDE>(p, row, SIDE == kBwdRowsQ ? 0 : it.src, lo0, hi0);
            bwd_interval<SIDE>(p, row, 1, lo1, hi1);
            float nl2_row = 0.f, c_row = 0.f;
            if (SIDE == kBwdRowsQ) {
                const uint32_t par = iw & 1u;
                const float* rowd = reinterpret_cast<const float*>(smem + SM::OFF_ROWD);
                wait_bar_warp(&rowd_full[par], (iw >> 1) & 1u, abort_flag, p.err);
                c_row = rowd[(par * 2 + 0) * kBwdRows + lrow];
                nl2_row = rowd[(par * 2 + 1) * kBwdRows + lrow];
                ptx::mbar_arrive(&rowd_empty[par]);
            }
            float usum = 0.f;
            for (int t = 0; t < it.nsub; ++t, ++n) {
                if (static_cast<int>(n & 1u) != w) continue;
                const uint32_t set = n % NSET;
                wait_bar_warp(&s_full[set], (n / NSET) & 1u, abort_flag, p.err);
                ptx::tc_fence_after();
                const BwdCol cr = bwd_col<SIDE>(it, t);
                const bool s1 = (SIDE == kBwdRowsQ) && cr.src == 1;
                const int cmin = (s1 ? lo1 : lo0) - cr.y;
                const int cmax = (s1 ? hi1 : hi0) - cr.y;
                const uint32_t ld_saddr = smem_base + SM::OFF_LD + (n % NST) * 2 * kBwdCols * 4;
                // The per-column lse / D of a rows-KV sub-tile come in by bulk copy with the
                // stage: observe the stage's barrier (already complete) before reading them.
                if (SIDE == kBwdRowsKV) wait_bar_warp(&col_full[n % NST], (n / NST) & 1u, abort_flag, p.err);
                usum += bwd_subtile<SIDE>(tmem_base + lane_off + set * 128, cmin, cmax, sl2, nl2_row, c_row,
                                          ld_saddr);
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                ptx::mbar_arrive(&p_full[set]);
            }
            // ------------------------------------------------------------ epilogue
            // The gradient tile goes to shared memory in the swizzled layout of its tensor map, the
            // accumulator is released, and one thread stores the tile with TMA (rows past L are
            // clipped by the map).
            const uint32_t ab = iw % NACC;
            const uint32_t acc = tmem_base + lane_off + ACC0 + ab * 2 * D;
            const int wtid = threadIdx.x - 128 - 128 * w;  // 0..127 within the warpgroup
            constexpr int UNITS_PER_CHUNK = C::RB / 16;
            if (SIDE == kBwdRowsQ && NACC == 1) {
                // Only the warpgroup that took the item's last sub-tile runs the epilogue; the other
                // hands over its sum of u and goes on with the next item (whose first sub-tile is
                // its own).  One accumulator set: the next item's accumulations wait for acc_free,
                // so neither warpgroup gets more than one item ahead of the epilogue, and the two
                // usum_ready slots and the one stage cannot be reused before they are read.
                const int par = iw & 1;
                const int w_late = static_cast<int>((n - 1u) & 1u);  // n: one past the item's last sub-tile
                if (w != w_late) {
                    xch[(par * 2 + w) * kBwdRows + lrow] = usum;
                    ptx::mbar_arrive(&usum_ready[par]);
                } else {
                    uint8_t* stage = smem + SM::OFF_STG;
                    wait_bar_warp(&usum_ready[par], (iw >> 1) & 1u, abort_flag, p.err);
                    // D_i - c_i = the sum of u over both warpgroups' sub-tiles.
                    const float du = usum + xch[(par * 2 + (1 - w)) * kBwdRows + lrow];
                    // the previous item's store (by either warpgroup) has finished reading the stage
                    wait_bar_warp(stg_free, (iw & 1u) ^ 1u, abort_flag, p.err);
                    wait_bar_warp(&acc_full[ab], (iw / NACC) & 1u, abort_flag, p.err);
                    ptx::tc_fence_after();
                    constexpr int CW = D < 32 ? D : 32;
#pragma unroll
                    for (int c0 = 0; c0 < D; c0 += CW) {
                        float y[CW], x[CW];
                        load_tmem_cols<CW>(acc + c0, y);
                        load_tmem_cols<CW>(acc + D + c0, x);
#pragma unroll
                        for (int c = 0; c < CW; ++c) x[c] = fmaf(-du, y[c], x[c]);
#pragma unroll
                        for (int g = 0; g < CW / 8; ++g) {
                            const int unit = (c0 + 8 * g) / 8;
                            *reinterpret_cast<uint4*>(stage + (unit / UNITS_PER_CHUNK) * C::ROW_CHUNK +
                                                      swz_offset<C::RB>(lrow, unit % UNITS_PER_CHUNK)) =
                                pack8_bf16(&x[8 * g], p.scale);
                        }
                    }
                    ptx::tc_fence_before();
                    ptx::mbar_arrive_cnt(&acc_free[ab], 2);  // both warpgroups' share
                    {
                        const size_t r = static_cast<size_t>(it.row_z) * p.Lpad + row;
                        p.ws_nl2[r] = valid ? nl2_row : -INFINITY;
                        p.ws_D[r] = valid ? -(c_row + du) : 0.f;
                    }
                    ptx::fence_proxy_async_smem();
                    ptx::named_barrier_sync(2 + w, 128);
                    if (wtid == 0) {
                        for (int ch = 0; ch < C::NCH; ++ch)
                            ptx::tma_store_3d(&p.tm_ga[0], stage + ch * C::ROW_CHUNK, ch * (C::RB / 2), it.row0,
                                              it.row_z);
                        ptx::tma_store_commit();
                        ptx::tma_store_wait_read_all();
                        ptx::mbar_arrive(stg_free);
                    }
                }
            } else if (SIDE == kBwdRowsQ) {
                uint8_t* stage = smem + SM::OFF_STG;
                // the previous item's store has finished reading the stage
                if (w == 0 && wtid == 0) ptx::tma_store_wait_read_all();
                // D_i - c_i = the sum of u over both warpgroups' sub-tiles.
                const int par = iw & 1;
                xch[(par * 2 + w) * kBwdRows + lrow] = usum;
                ptx::named_barrier_sync(1, kSoftmaxThreads);
                const float du = xch[(par * 2 + 0) * kBwdRows + lrow] + xch[(par * 2 + 1) * kBwdRows + lrow];
                wait_bar_warp(&acc_full[ab], (iw / NACC) & 1u, abort_flag, p.err);
                ptx::tc_fence_after();
                constexpr int HALF = D / 2;
                constexpr int CW = HALF < 32 ? HALF : 32;
#pragma unroll
                for (int c0 = w * HALF; c0 < (w + 1) * HALF; c0 += CW) {
                    float y[CW], x[CW];
                    load_tmem_cols<CW>(acc + c0, y);
                    load_tmem_cols<CW>(acc + D + c0, x);
#pragma unroll
                    for (int c = 0; c < CW; ++c) x[c] = fmaf(-du, y[c], x[c]);
#pragma unroll
                    for (int g = 0; g < CW / 8; ++g) {
                        const int unit = (c0 + 8 * g) / 8;
                        *reinterpret_cast<uint4*>(stage + (unit / UNITS_PER_CHUNK) * C::ROW_CHUNK +
                                                  swz_offset<C::RB>(lrow, unit % UNITS_PER_CHUNK)) =
                            pack8_bf16(&x[8 * g], p.scale);
                    }
                }
                ptx::tc_fence_before();
                ptx::mbar_arrive(&acc_free[ab]);
                if (w == 0) {
                    const size_t r = static_cast<size_t>(it.row_z) * p.Lpad + row;
                    p.ws_nl2[r] = valid ? nl2_row : -INFINITY;
                    p.ws_D[r] = valid ? -(c_row + du) : 0.f;
                }
                ptx::fence_proxy_async_smem();
                ptx::named_barrier_sync(1, kSoftmaxThreads);
                if (w == 0 && wtid == 0) {
                    for (int ch = 0; ch < C::NCH; ++ch)
                        ptx::tma_store_3d(&p.tm_ga[0], stage + ch * C::ROW_CHUNK, ch * (C::RB / 2), it.row0,
                                          it.row_z);
                    ptx::tma_store_commit();
                }
            } else {
                // warpgroup 0 writes dv = dV, warpgroup 1 dk = scale dK, each from its own stage
                uint8_t* stage = smem + SM::OFF_STG + w * C::ROW_TILE;
                if (wtid == 0) ptx::tma_store_wait_read_all();
                ptx::named_barrier_sync(2 + w, 128);
                wait_bar_warp(&acc_full[ab], (iw / NACC) & 1u, abort_flag, p.err);
                ptx::tc_fence_after();
                constexpr int CW = D < 32 ? D : 32;
                const float f = (w == 0) ? 1.f : p.scale;
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += CW) {
                    float v[CW];
                    load_tmem_cols<CW>(acc + w * D + c0, v);
#pragma unroll
                    for (int g = 0; g < CW / 8; ++g) {
                        const int unit = (c0 + 8 * g) / 8;
                        *reinterpret_cast<uint4*>(stage + (unit / UNITS_PER_CHUNK) * C::ROW_CHUNK +
                                                  swz_offset<C::RB>(lrow, unit % UNITS_PER_CHUNK)) =
                            pack8_bf16(&v[8 * g], f);
                    }
                }
                ptx::tc_fence_before();
                ptx::mbar_arrive(&acc_free[ab]);
                ptx::fence_proxy_async_smem();
                ptx::named_barrier_sync(2 + w, 128);
                if (wtid == 0) {
                    const CUtensorMap* m = (w == 0) ? &p.tm_ga[it.src] : &p.tm_gb[it.src];
                    for (int ch = 0; ch < C::NCH; ++ch)
                        ptx::tma_store_3d(m, stage + ch * C::ROW_CHUNK, ch * (C::RB / 2), it.row0, it.row_z);
                    ptx::tma_store_commit();
                }
            }
            ++iw;
        }
        // every issued store has completed before the CTA exits
        if (threadIdx.x == 128 || threadIdx.x == 256) ptx::tma_store_wait_all();
        ptx::tc_fence_before();
        ptx::mbar_arrive(softmax_done);
    }
#undef E2D2_BWD_SMEM_POINTERS
}

}  // namespace e2d2
