// fmha_sm100.cuh -- persistent, warp-specialised flash attention for B200 (sm_100a) that
// computes the three E2D2 attention calls:
//
//   kEncoder        block-causal self-attention over clean tokens: query i sees keys j with
//                   floor(j/S) <= floor(i/S)  ("Encoder-Decoder Diffusion Language Models for
//                   Efficient Training and Inference", paper notes, sec. 4).
//   kDecoderTrain   fused self+cross attention over 2L keys: encoder-side keys of the blocks
//                   strictly before the query's block, decoder-side keys of its own block
//                   (same page, sec. 2 and 4).
//   kDecoderSample  sampling step: the S noised queries of one block (G = Hq/Hkv heads packed
//                   into the rows of one tile) against the cached clean prefix (P keys) and
//                   their own block (same page, sec. 3), split over CTAs stream-K style.
//
// Every row's allowed keys form, per key source, one interval [lo, hi), so the mask is
// computed from tile indices and row numbers; key tiles outside every row's interval are
// never loaded, and no mask matrix exists anywhere.
//
// CTA = 10 warps: warp 0 issues TMA loads, warp 1 owns tensor memory and issues tcgen05.mma,
// warps 2..9 run the online softmax and the epilogue.  One 128-row query tile per work item;
// per key tile of up to 128 keys:
//     S   = Q K^T          tcgen05.mma, A = Q (smem), B = K (smem, K-major)  -> TMEM (fp32)
//     P   = exp2(S*c - m)  softmax warps, written back over S as bf16      -> TMEM
//     O_h += P_h V_h       tcgen05.mma, A = P (TMEM), B = V (smem, MN-major) -> TMEM (fp32)
// The key columns of every tile are split in two halves h (keys 0-63 and 64-127).  Each half
// has its own softmax warps (the two warps on one TMEM lane quarter: same rows, different
// keys), its own running max m_h and sum l_h, and its own accumulator O_h; the halves are
// merged once, in the epilogue (O = sum_h 2^(m_h - M) O_h / sum_h 2^(m_h - M) l_h).  So the
// two warps never wait for each other inside the key loop, and the tensor core gets two
// independent P.V accumulation chains to interleave.
// S is double-buffered in TMEM so QK^T of tile j+1 overlaps the softmax of tile j; at
// head_dim <= 64 the O pair is double-buffered across work items as well.  A running max is
// only moved when it grows by more than 2^8 (log2 units), so O is rescaled rarely; the final
// normalisation uses the same max and is exact.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx_sm100.cuh"

namespace e2d2 {

enum Mode : int { kEncoder = 0, kDecoderTrain = 1, kDecoderSample = 2 };

constexpr int kBlockM = 128;            // query rows per tile (TMEM lanes)
constexpr int kBlockN = 128;            // keys per tile
constexpr int kThreads = 320;           // 10 warps
constexpr int kSoftmaxThreads = 256;    // warps 2..9
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;
constexpr int kSampleMaxCtas = 256;     // upper bound of the sampling grid (workspace sizing)
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s per wait

// Bit set in the device error word when a bounded wait gives up.
constexpr unsigned int kErrWaitTimeout = 1u;

struct alignas(64) FmhaParams {
    CUtensorMap tm_q;   // kEncoder/kDecoderTrain: 3D {D, L, B*Hq}; kDecoderSample: 2D {D, B*Hq*S}
    CUtensorMap tm_k0;  // source 0: encoder self K | decoder-train encoder-side K | sample cache K
    CUtensorMap tm_v0;
    CUtensorMap tm_k1;  // source 1: decoder-train decoder-side K | sample own-block K
    CUtensorMap tm_v1;
    CUtensorMap tm_o;   // train modes: 3D {D, L, B*Hq} (TMA store)
    void* out;          // kDecoderSample output, bf16 [B][Hq][S][D]
    float* lse;         // nullable
    float* ws_partial;  // kDecoderSample: split partial slots
    int* ws_tickets;    // kDecoderSample: one ticket word per CTA
    unsigned int* err;  // device error word
    int batch, q_heads, kv_heads, group;
    int L;              // train: sequence length
    int S;              // block size
    int P;              // sample: cached prefix length
    int box1_rows;      // rows of one source-1 TMA box
    float scale_log2;   // softmax scale * log2(e)
    int num_items;      // train: (head, query tile) items
    int num_qtiles;     // train: query tiles per head; sample: query tiles per (b, kv head)
    int rows_per_unit;  // sample: G * S packed query rows per (b, kv head)
    int tiles_per_unit; // sample: key tiles per unit
    long long total_tiles;  // sample: units * tiles_per_unit
    int slot_floats;    // sample: floats per partial slot
    int rows_cap;       // sample: rows stored per partial slot
};

// A unit of work: one 128-row query tile against a contiguous range of its key tiles.
struct Item {
    int q_z;        // train: b*Hq + h (Q/O tensor-map z); sample: unit index
    int kv_z;       // b*Hkv + g
    int q_row0;     // train: first row within the head; sample: first packed row within the unit
    int q_y;        // TMA y coordinate of the query tile
    int out_row0;   // sample: first row of this tile in the [B*Hq*S] row space
    int n1, a1;     // source-1 tiles (visited first), starting at key tile a1
    int n0;         // source-0 tiles, starting at key tile 0
    int t_begin, t_end;
};

template <int D>
struct Cfg {
    static constexpr int NOB = (D <= 64) ? 2 : 1;             // O accumulator sets in TMEM
    static constexpr int RB = (D * 2 < 128) ? D * 2 : 128;  // bytes per smem row of one chunk
    static constexpr int NCH = D * 2 / RB;                   // column chunks per tile
    static constexpr uint32_t SWZ = (RB == 128) ? 2u : 4u;   // 128-byte / 64-byte swizzle
    static constexpr int CHUNK_BYTES = kBlockM * RB;
    static constexpr int TILE_BYTES = kBlockM * D * 2;
    static constexpr int NST = (D == 128) ? 2 : (D == 64 ? 4 : 6);
    static constexpr int KSTEPS_PER_CHUNK = RB / 32;         // 16-element k steps per chunk
};

template <int D, int MODE>
struct Smem {
    using C = Cfg<D>;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + 2 * C::TILE_BYTES;
    static constexpr int OFF_V = OFF_K + C::NST * C::TILE_BYTES;
    static constexpr int OFF_O = OFF_V + C::NST * C::TILE_BYTES;
    // Train calls stage the output tile for a TMA store, except at d = 128 where the shared
    // memory is taken by the K/V ring; there rows are stored directly.
    static constexpr bool STAGE_O = (MODE != kDecoderSample) && (D <= 64);
    static constexpr int O_BYTES = STAGE_O ? C::TILE_BYTES : 0;
    static constexpr int OFF_BAR = OFF_O + O_BYTES;
    // barriers: k_full[NST], v_full[NST], kv_empty[NST], q_full[2], q_empty[2], s_full[2],
    // p_full[2 S buffers][2 halves], o_free[2], pv_done[2 halves], mma_drain
    static constexpr int NBAR = 3 * C::NST + 2 + 2 + 2 + 4 + 2 + 2 + 1;
    static constexpr int OFF_RED = ((OFF_BAR + NBAR * 8 + 15) / 16) * 16;  // per-half (m, l) exchange
    static constexpr int OFF_MISC = OFF_RED + 4 * kBlockM * 4;
    static constexpr int BYTES = OFF_MISC + 64;
    static constexpr int ALLOC = ((BYTES + 1023) / 1024) * 1024 + 1024;  // + alignment slack
};

__device__ __forceinline__ int ceil_div_i(int a, int b) { return (a + b - 1) / b; }
__device__ __forceinline__ int round16(int x) { return (x + 15) & ~15; }

// Largest CTA c whose stream-K range [c*T/G, (c+1)*T/G) starts at or before tile x.
__device__ __forceinline__ int owner_cta(long long x, long long T, int grid) {
    return static_cast<int>(((x + 1) * grid - 1) / T);
}
__device__ __forceinline__ long long range_begin(int c, long long T, int grid) {
    return (static_cast<long long>(c) * T) / grid;
}

// Iterates the work items of this CTA.  Every role walks the same sequence.
template <int MODE>
struct Scheduler {
    const FmhaParams& p;
    long long pos, end;  // sample: tile range of this CTA
    int k;               // train: next item index

    __device__ Scheduler(const FmhaParams& prm) : p(prm) {
        if (MODE == kDecoderSample) {
            pos = range_begin(blockIdx.x, p.total_tiles, gridDim.x);
            end = range_begin(blockIdx.x + 1, p.total_tiles, gridDim.x);
        } else {
            k = blockIdx.x;
        }
    }

    __device__ bool next(Item& it) {
        if (MODE == kDecoderSample) {
            if (pos >= end) return false;
            const int Tu = p.tiles_per_unit;
            const int u = static_cast<int>(pos / Tu);
            const long long ubeg = static_cast<long long>(u) * Tu;
            const long long seg_end = (end < ubeg + Tu) ? end : ubeg + Tu;
            const int qt = u % p.num_qtiles;
            const int kvz = u / p.num_qtiles;  // b*Hkv + g
            const int b = kvz / p.kv_heads, g = kvz % p.kv_heads;
            it.q_z = u;
            it.kv_z = kvz;
            it.q_row0 = qt * kBlockM;
            it.out_row0 = (b * p.q_heads + g * p.group) * p.S + qt * kBlockM;
            it.q_y = it.out_row0;
            it.n1 = ceil_div_i(p.S, kBlockN);
            it.a1 = 0;
            it.n0 = ceil_div_i(p.P, kBlockN);
            it.t_begin = static_cast<int>(pos - ubeg);
            it.t_end = static_cast<int>(seg_end - ubeg);
            pos = seg_end;
            return true;
        } else {
            if (k >= p.num_items) return false;
            const int BH = p.batch * p.q_heads;
            const int qt = p.num_qtiles - 1 - k / BH;  // longest rows first
            const int bh = k % BH;
            k += gridDim.x;
            const int b = bh / p.q_heads, h = bh % p.q_heads;
            it.q_z = bh;
            it.kv_z = b * p.kv_heads + h / p.group;
            it.q_row0 = qt * kBlockM;
            it.q_y = it.q_row0;
            it.out_row0 = 0;
            const int L = p.L, S = p.S;
            const int q_last = min(L, it.q_row0 + kBlockM) - 1;
            if (MODE == kEncoder) {
                const int hi = min(L, (q_last / S + 1) * S);
                it.n1 = 0;
                it.a1 = 0;
                it.n0 = ceil_div_i(hi, kBlockN);
            } else {
                const int own_lo = (it.q_row0 / S) * S;
                const int own_hi = min(L, (q_last / S + 1) * S);
                it.a1 = own_lo / kBlockN;
                it.n1 = ceil_div_i(own_hi, kBlockN) - it.a1;
                it.n0 = ceil_div_i((q_last / S) * S, kBlockN);
            }
            it.t_begin = 0;
            it.t_end = it.n1 + it.n0;
            return true;
        }
    }
};

// Virtual tile t of an item -> (source, key tile, keys in the tile rounded to 16, box rows).
struct TileRef {
    int src, kt, nk16, box_rows;
};

template <int MODE>
__device__ __forceinline__ TileRef tile_of(const FmhaParams& p, const Item& it, int t) {
    TileRef r;
    if (t < it.n1) {
        r.src = 1;
        r.kt = it.a1 + t;
        const int len = (MODE == kDecoderSample) ? p.S : p.L;
        r.nk16 = round16(min(kBlockN, len - r.kt * kBlockN));
        r.box_rows = p.box1_rows;
    } else {
        r.src = 0;
        r.kt = t - it.n1;
        const int len = (MODE == kDecoderSample) ? p.P : p.L;
        r.nk16 = round16(min(kBlockN, len - r.kt * kBlockN));
        r.box_rows = kBlockN;
    }
    return r;
}

// Bounded mbarrier wait.  Returns false (and flags the CTA and the device error word) if the
// phase does not complete within kWaitTimeoutNs or another role already gave up.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         unsigned int* err) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t spin = 1;; ++spin) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((spin & 255u) == 0) {
            if (*abort_flag) return false;
            if (ptx::globaltimer_ns() - t0 > kWaitTimeoutNs) {
                *abort_flag = 1;
                atomicOr(err, kErrWaitTimeout);
                return false;
            }
        }
    }
}

// Warp-collective form of wait_bar: every lane returns the same answer, so the .sync.aligned
// tcgen05 instructions that follow are always executed by the whole warp.
__device__ __forceinline__ bool wait_bar_warp(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              unsigned int* err) {
    const bool ok = wait_bar(bar, parity, abort_flag, err);
    return __all_sync(0xffffffffu, ok);
}

// Byte offset of 16-byte unit `u` of row `r` inside one swizzled chunk (row pitch RB bytes).
template <int RB>
__device__ __forceinline__ uint32_t swz_offset(int r, int u) {
    const uint32_t a = static_cast<uint32_t>(r * RB + u * 16);
    constexpr uint32_t mask = (RB == 128) ? 7u : 3u;
    return a ^ (((a >> 7) & mask) << 4);
}

// Issues the two P.V chains of one key tile: O[ob][h] += P[sb][keys of half h] . V[st][same keys]
// (A = P read from TMEM, B = V MN-major in shared memory), interleaved so the tensor core always
// has an independent accumulation to work on.  Waits for both halves' P (p_full), for the O set
// to be free (first tile of an item), and for V.  State is passed by value (nothing in local
// memory).  started[h]: chain h already holds a partial sum in this item.
template <class C>
__device__ __forceinline__ bool issue_pv(uint64_t* p_full, uint64_t* o_free, uint64_t* v_full,
                                         uint64_t* kv_empty, uint64_t* pv_done, volatile int* abort_flag,
                                         unsigned int* err, uint32_t tmem_base, uint32_t sV, uint64_t vdesc,
                                         uint32_t idesc_pv, uint32_t sb, uint32_t st, uint32_t round,
                                         uint32_t g, uint32_t ob, uint32_t item, uint32_t nk, bool first,
                                         int D, bool (&started)[2], bool leader) {
    if (!wait_bar_warp(&p_full[2 * sb + 0], (g >> 1) & 1, abort_flag, err)) return false;
    if (!wait_bar_warp(&p_full[2 * sb + 1], (g >> 1) & 1, abort_flag, err)) return false;
    if (first && !wait_bar_warp(&o_free[ob], ((item / C::NOB) & 1) ^ 1, abort_flag, err)) return false;
    if (!wait_bar_warp(&v_full[st], round & 1, abort_flag, err)) return false;
    ptx::tc_fence_after();
    const uint32_t a_tmem = tmem_base + sb * 128;
    const uint32_t v_base = sV + st * C::TILE_BYTES;
    const uint32_t nks = nk / 16;  // 16-key steps in this tile; half h owns steps [4h, 4h+4)
    if (leader) {
#pragma unroll
        for (uint32_t i = 0; i < 4; ++i) {
#pragma unroll
            for (uint32_t h = 0; h < 2; ++h) {
                const uint32_t ks = 4 * h + i;
                if (ks < nks) {
                    const uint32_t d_tmem = tmem_base + 256 + (ob * 2 + h) * D;
                    // P of half h sits in the first 32 of that half's own 64 S columns.
                    ptx::mma_ts(d_tmem, a_tmem + 64 * h + i * 8, vdesc | ((v_base + ks * 16 * C::RB) >> 4),
                                idesc_pv, (started[h] || i > 0) ? 1u : 0u);
                }
            }
        }
        ptx::mma_commit(&pv_done[0]);
        ptx::mma_commit(&pv_done[1]);
        ptx::mma_commit(&kv_empty[st]);
    }
    __syncwarp();
    if (nks > 0) started[0] = true;
    if (nks > 4) started[1] = true;
    return true;
}

// Loads N consecutive fp32 TMEM columns of this thread's lane (N in {16, 32, 64}).
template <int N>
__device__ __forceinline__ void load_tmem_cols(uint32_t taddr, float* o) {
    uint32_t r[N];
    if constexpr (N == 16) {
        ptx::tmem_ld16(taddr, *reinterpret_cast<uint32_t(*)[16]>(r));
    } else {
#pragma unroll
        for (int c = 0; c < N; c += 32) ptx::tmem_ld32(taddr + c, &r[c]);
    }
    ptx::tmem_wait_ld();
    ptx::reg_fence<N>(r);
#pragma unroll
    for (int c = 0; c < N; ++c) o[c] = __uint_as_float(r[c]);
}

// Multiplies N consecutive fp32 TMEM columns of this thread's lane by f.
template <int N>
__device__ __forceinline__ void rescale_tmem_cols(uint32_t taddr, float f) {
    constexpr int W = N < 32 ? N : 32;
#pragma unroll
    for (int c0 = 0; c0 < N; c0 += W) {
        uint32_t r[W];
        if constexpr (W == 16) {
            ptx::tmem_ld16(taddr + c0, *reinterpret_cast<uint32_t(*)[16]>(r));
        } else {
            ptx::tmem_ld32(taddr + c0, r);
        }
        ptx::tmem_wait_ld();
        ptx::reg_fence<W>(r);
#pragma unroll
        for (int c = 0; c < W; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * f);
        if constexpr (W == 16) {
            ptx::tmem_st16(taddr + c0, r);
        } else {
            ptx::tmem_st32(taddr + c0, r);
        }
    }
}

__device__ __forceinline__ uint4 pack8_bf16(const float* v, float scale) {
    uint4 w;
    w.x = ptx::pack_bf16x2(v[0] * scale, v[1] * scale);
    w.y = ptx::pack_bf16x2(v[2] * scale, v[3] * scale);
    w.z = ptx::pack_bf16x2(v[4] * scale, v[5] * scale);
    w.w = ptx::pack_bf16x2(v[6] * scale, v[7] * scale);
    return w;
}

template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, 1) fmha_sm100_kernel(const __grid_constant__ FmhaParams p) {
    using C = Cfg<D>;
    using SM = Smem<D, MODE>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::OFF_BAR);
    uint64_t* k_full = bars;
    uint64_t* v_full = bars + C::NST;
    uint64_t* kv_empty = bars + 2 * C::NST;
    uint64_t* q_full = bars + 3 * C::NST;
    uint64_t* q_empty = q_full + 2;
    uint64_t* s_full = q_full + 4;
    uint64_t* p_full = q_full + 6;    // [sb][half]
    uint64_t* o_free = q_full + 10;   // [ob]
    uint64_t* pv_done = q_full + 12;  // [half]
    uint64_t* mma_drain = q_full + 14;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SM::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM::OFF_MISC + 8);
    volatile int* bcast = reinterpret_cast<volatile int*>(smem + SM::OFF_MISC + 16);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NST; ++i) {
            ptx::mbar_init(&k_full[i], 1);
            ptx::mbar_init(&v_full[i], 1);
            ptx::mbar_init(&kv_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&q_full[i], 1);
            ptx::mbar_init(&q_empty[i], 1);
            ptx::mbar_init(&s_full[i], 1);
            ptx::mbar_init(&o_free[i], kSoftmaxThreads);
            ptx::mbar_init(&pv_done[i], 1);
        }
        for (int i = 0; i < 4; ++i) ptx::mbar_init(&p_full[i], kSoftmaxThreads / 2);
        ptx::mbar_init(mma_drain, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_holder, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    const uint32_t smem_base = ptx::smem_u32(smem);
    const uint32_t sQ = smem_base + SM::OFF_Q;
    const uint32_t sK = smem_base + SM::OFF_K;
    const uint32_t sV = smem_base + SM::OFF_V;

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        // The whole warp walks the schedule (warp-uniform control flow); one elected lane
        // issues the copies.
        const bool leader = ptx::elect_one();
        if (leader) {
            ptx::tma_prefetch_desc(&p.tm_q);
            ptx::tma_prefetch_desc(&p.tm_k0);
            ptx::tma_prefetch_desc(&p.tm_v0);
            if (MODE != kEncoder) {
                ptx::tma_prefetch_desc(&p.tm_k1);
                ptx::tma_prefetch_desc(&p.tm_v1);
            }
        }
        __syncwarp();
        Scheduler<MODE> sched(p);
        Item it;
        uint32_t kv_iter = 0, item_idx = 0;
        bool ok = true;
        while (ok && sched.next(it)) {
            const int qb = item_idx & 1;
            const uint32_t qround = item_idx >> 1;
            ok = wait_bar_warp(&q_empty[qb], (qround & 1) ^ 1, abort_flag, p.err);
            if (!ok) break;
            if (leader) {
                ptx::mbar_arrive_expect_tx(&q_full[qb], C::TILE_BYTES);
                for (int ch = 0; ch < C::NCH; ++ch) {
                    uint8_t* dst = smem + SM::OFF_Q + qb * C::TILE_BYTES + ch * C::CHUNK_BYTES;
                    if (MODE == kDecoderSample)
                        ptx::tma_load_2d(&p.tm_q, &q_full[qb], dst, ch * (C::RB / 2), it.q_y);
                    else
                        ptx::tma_load_3d(&p.tm_q, &q_full[qb], dst, ch * (C::RB / 2), it.q_y, it.q_z);
                }
            }
            __syncwarp();
            ++item_idx;
            for (int t = it.t_begin; t < it.t_end; ++t) {
                const int st = kv_iter % C::NST;
                const uint32_t round = kv_iter / C::NST;
                ok = wait_bar_warp(&kv_empty[st], (round & 1) ^ 1, abort_flag, p.err);
                if (!ok) break;
                const TileRef tr = tile_of<MODE>(p, it, t);
                if (leader) {
                    const CUtensorMap* mk = tr.src ? &p.tm_k1 : &p.tm_k0;
                    const CUtensorMap* mv = tr.src ? &p.tm_v1 : &p.tm_v0;
                    const uint32_t bytes = static_cast<uint32_t>(tr.box_rows) * D * 2;
                    ptx::mbar_arrive_expect_tx(&k_full[st], bytes);
                    for (int ch = 0; ch < C::NCH; ++ch)
                        ptx::tma_load_3d(mk, &k_full[st],
                                         smem + SM::OFF_K + st * C::TILE_BYTES + ch * C::CHUNK_BYTES,
                                         ch * (C::RB / 2), tr.kt * kBlockN, it.kv_z);
                    ptx::mbar_arrive_expect_tx(&v_full[st], bytes);
                    for (int ch = 0; ch < C::NCH; ++ch)
                        ptx::tma_load_3d(mv, &v_full[st],
                                         smem + SM::OFF_V + st * C::TILE_BYTES + ch * C::CHUNK_BYTES,
                                         ch * (C::RB / 2), tr.kt * kBlockN, it.kv_z);
                }
                __syncwarp();
                ++kv_iter;
            }
        }
        // Never leave with copies in flight: wait for the last load of every buffer (the last
        // NST K/V loads and the last two Q loads).
        volatile int no_abort = 0;
        const uint32_t first_live = kv_iter > static_cast<uint32_t>(C::NST) ? kv_iter - C::NST : 0u;
        for (uint32_t i = first_live; i < kv_iter; ++i) {
            wait_bar_warp(&k_full[i % C::NST], (i / C::NST) & 1u, &no_abort, p.err);
            wait_bar_warp(&v_full[i % C::NST], (i / C::NST) & 1u, &no_abort, p.err);
        }
        for (uint32_t i = item_idx > 2u ? item_idx - 2u : 0u; i < item_idx; ++i)
            wait_bar_warp(&q_full[i & 1u], (i >> 1) & 1u, &no_abort, p.err);
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        // The whole warp walks the schedule, so descriptors and TMEM addresses are warp-uniform;
        // one elected lane issues tcgen05.mma / tcgen05.commit.
        const bool leader = ptx::elect_one();
        Scheduler<MODE> sched(p);
        Item it;
        uint32_t kv_iter = 0, gtile = 0, item_idx = 0;
        // Descriptor bits without the start address (added per MMA).
        const uint64_t kdesc = ptx::smem_desc(0, 16, 8 * C::RB, C::SWZ);             // Q, K: K-major
        const uint64_t vdesc = ptx::smem_desc(0, C::CHUNK_BYTES, 8 * C::RB, C::SWZ);  // V: MN-major
        constexpr uint32_t idesc_pv = ptx::idesc_bf16_f32(kBlockM, D, true);
        // The P.V of tile j is issued after the QK^T of tile j+1, so the tensor core computes
        // S_{j+1} while the softmax warps work on tile j.
        bool have_pv = false, pv_first = false;
        bool started[2] = {false, false};  // chains of the item the pending P.V belongs to
        uint32_t pv_sb = 0, pv_st = 0, pv_round = 0, pv_g = 0, pv_ob = 0, pv_item = 0, pv_nk = 0;
        bool ok = true;
        while (ok && sched.next(it)) {
            const int qb = item_idx & 1;
            ok = wait_bar_warp(&q_full[qb], (item_idx >> 1) & 1, abort_flag, p.err);
            if (!ok) break;
            const uint32_t q_base = sQ + qb * C::TILE_BYTES;
            if (it.t_end <= it.t_begin && leader) ptx::mma_commit(&q_empty[qb]);
            for (int t = it.t_begin; t < it.t_end; ++t) {
                const uint32_t st = kv_iter % C::NST;
                const uint32_t round = kv_iter / C::NST;
                ok = wait_bar_warp(&k_full[st], round & 1, abort_flag, p.err);
                if (!ok) break;
                ptx::tc_fence_after();
                const TileRef tr = tile_of<MODE>(p, it, t);
                const uint32_t sb = gtile & 1;
                const uint32_t idesc_qk = ptx::idesc_bf16_f32(kBlockM, tr.nk16, false);
                const uint32_t k_base = sK + st * C::TILE_BYTES;
                if (leader) {
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t off = (ks / C::KSTEPS_PER_CHUNK) * C::CHUNK_BYTES +
                                             (ks % C::KSTEPS_PER_CHUNK) * 32;
                        ptx::mma_ss(tmem_base + sb * 128, kdesc | ((q_base + off) >> 4),
                                    kdesc | ((k_base + off) >> 4), idesc_qk, ks > 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(&s_full[sb]);
                    if (t == it.t_end - 1) ptx::mma_commit(&q_empty[qb]);
                }
                __syncwarp();
                if (have_pv) {
                    ok = issue_pv<C>(p_full, o_free, v_full, kv_empty, pv_done, abort_flag, p.err, tmem_base, sV,
                                     vdesc, idesc_pv, pv_sb, pv_st, pv_round, pv_g, pv_ob, pv_item, pv_nk,
                                     pv_first, D, started, leader);
                    if (!ok) break;
                }
                // started[] follows the item of the pending P.V: a new item starts both chains afresh.
                if (t == it.t_begin) started[0] = started[1] = false;
                have_pv = true;
                pv_sb = sb;
                pv_st = st;
                pv_round = round;
                pv_g = gtile;
                pv_ob = item_idx % C::NOB;
                pv_item = item_idx;
                pv_nk = tr.nk16;
                pv_first = (t == it.t_begin);
                ++kv_iter;
                ++gtile;
            }
            ++item_idx;
        }
        if (ok && have_pv)
            issue_pv<C>(p_full, o_free, v_full, kv_empty, pv_done, abort_flag, p.err, tmem_base, sV, vdesc,
                        idesc_pv, pv_sb, pv_st, pv_round, pv_g, pv_ob, pv_item, pv_nk, pv_first, D, started,
                        leader);
        // Drain: every MMA issued by this warp completes before TMEM is released.
        if (leader) ptx::mma_commit(mma_drain);
        __syncwarp();
        volatile int no_abort = 0;
        wait_bar_warp(mma_drain, 0, &no_abort, p.err);
    } else {
        // ------------------------------------------------------------------ softmax warps
        // Eight warps.  Warps w and w+4 share TMEM lane quarter (w & 3) -- the same 32 query
        // rows -- and own the two key halves of every S tile (keys 0-63 / 64-127) with their
        // own running max, sum and O accumulator.  They meet only in the epilogue.  Waits never
        // break these loops: every warp takes every named barrier, so a wait that gives up
        // (device error word set) cannot strand another warp.
        const int sw = warp - 2;                     // 0..7
        const int half = sw >> 2;                    // key half of this thread
        const int quarter = warp & 3;                // TMEM lane quarter
        const int row = quarter * 32 + lane;         // query row of the tile
        const int stid = threadIdx.x - 64;           // 0..255 within the softmax group
        const uint32_t pair_bar = 2 + quarter;       // named barrier of the two warps of a quarter
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        constexpr int DH = D / 2;                    // output columns written by this thread
        float* xch = reinterpret_cast<float*>(smem + SM::OFF_RED);  // [m|l][half][128]
        const float sl2 = p.scale_log2;
        Scheduler<MODE> sched(p);
        Item it;
        uint32_t gtile = 0, item_idx = 0;
        while (sched.next(it)) {
            // Per-row key intervals [lo, hi) for source 0 and source 1 (empty for padded rows).
            int lo0, hi0, lo1, hi1;
            bool row_valid;
            if (MODE == kDecoderSample) {
                row_valid = (it.q_row0 + row) < p.rows_per_unit;
                lo0 = 0;
                hi0 = row_valid ? p.P : 0;
                lo1 = 0;
                hi1 = row_valid ? p.S : 0;
            } else {
                const int i_raw = it.q_row0 + row;
                row_valid = i_raw < p.L;
                const int i = min(i_raw, p.L - 1);
                const int b0 = (i / p.S) * p.S;
                if (MODE == kEncoder) {
                    lo0 = 0;
                    hi0 = row_valid ? min(p.L, b0 + p.S) : 0;
                    lo1 = 0;
                    hi1 = 0;
                } else {
                    lo0 = 0;
                    hi0 = row_valid ? b0 : 0;
                    lo1 = b0;
                    hi1 = row_valid ? min(p.L, b0 + p.S) : 0;
                }
            }
            float m = -INFINITY, l = 0.f;  // this half's running max (log2 units) and sum
            const uint32_t ob = item_idx % C::NOB;
            const uint32_t o_base = tmem_base + lane_off + 256 + ob * 2 * D;  // O[ob][0]; O[ob][1] at +D
            const uint32_t o_mine = o_base + half * D;
            for (int t = it.t_begin; t < it.t_end; ++t) {
                const uint32_t sb = gtile & 1;
                wait_bar_warp(&s_full[sb], (gtile >> 1) & 1, abort_flag, p.err);
                ptx::tc_fence_after();
                const TileRef tr = tile_of<MODE>(p, it, t);
                const int k0 = tr.kt * kBlockN;
                const int lo = tr.src ? lo1 : lo0;
                const int hi = tr.src ? hi1 : hi0;
                const int cmin = lo - k0;
                const int cmax = min(hi - k0, tr.nk16);
                const int nchunks = (tr.nk16 + 31) / 32;
                const uint32_t s_tmem = tmem_base + lane_off + sb * 128;
                // This thread's chunks are a = 2*half + cc.  live: some row of the warp has an
                // allowed key in the chunk (warp-uniform).
                uint32_t live = 0;
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int a = 2 * half + cc;
                    const bool mine = (a < nchunks) && (cmin < 32 * a + 32) && (cmax > 32 * a);
                    if (__any_sync(0xffffffffu, mine)) live |= 1u << cc;
                }
                uint32_t s_raw[64];
#pragma unroll
                for (int cc = 0; cc < 2; ++cc)
                    if (live & (1u << cc)) ptx::tmem_ld32(s_tmem + 32 * (2 * half + cc), &s_raw[32 * cc]);
                ptx::tmem_wait_ld();
                ptx::reg_fence<64>(s_raw);
                float s[64];
#pragma unroll
                for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(s_raw[c]);
                float cmx[2] = {-INFINITY, -INFINITY};
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    if (live & (1u << cc)) {
                        const int a = 2 * half + cc;
                        const bool whole = (cmin <= 32 * a) && (cmax >= 32 * a + 32);
                        if (!__all_sync(0xffffffffu, whole)) {
#pragma unroll
                            for (int c = 0; c < 32; ++c) {
                                const int col = 32 * a + c;
                                s[32 * cc + c] = (col >= cmin && col < cmax) ? s[32 * cc + c] : -INFINITY;
                            }
                        }
#pragma unroll
                        for (int c = 0; c < 32; c += 2)
                            cmx[cc] = ptx::fmax3(cmx[cc], s[32 * cc + c], s[32 * cc + c + 1]);
                    }
                }
                const float m_new = fmaxf(m, fmaxf(cmx[0], cmx[1]) * sl2);
                const bool first = (t == it.t_begin);
                bool rescale = false;
                float alpha = 1.f;
                if (m_new > m + kRescaleThreshold) {
                    alpha = ptx::ex2(m - m_new);
                    rescale = !first;
                    m = m_new;
                    l *= alpha;
                }
                const float neg_m = (m == -INFINITY) ? 0.f : -m;
                // P = exp2(s * scale*log2e - m) in bf16, written over this half's own S columns
                // (which no other warp reads): keys 64h + 32cc .. +31 -> TMEM columns
                // 64h + 16cc .. +15.  Dead chunks are zeros.
                float sums[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int a = 2 * half + cc;
                    if (a < nchunks) {
                        uint32_t pk[16];
                        if (live & (1u << cc)) {
#pragma unroll
                            for (int c = 0; c < 32; c += 2) {
                                const float e0 = ptx::ex2(fmaf(s[32 * cc + c], sl2, neg_m));
                                const float e1 = ptx::ex2(fmaf(s[32 * cc + c + 1], sl2, neg_m));
                                sums[(c >> 1) & 3] += e0 + e1;
                                pk[c / 2] = ptx::pack_bf16x2(e0, e1);
                            }
                        } else {
#pragma unroll
                            for (int c = 0; c < 16; ++c) pk[c] = 0u;
                        }
                        ptx::tmem_st16(s_tmem + 64 * half + 16 * cc, pk);
                    }
                }
                l += (sums[0] + sums[1]) + (sums[2] + sums[3]);
                if (!first) {
                    // This half's O may only be touched once its previous P.V has landed.
                    wait_bar_warp(&pv_done[half], (gtile - 1) & 1, abort_flag, p.err);
                    ptx::tc_fence_after();
                    // tcgen05.ld/st are warp-collective: the warp rescales if any row needs it.
                    if (__any_sync(0xffffffffu, rescale)) rescale_tmem_cols<D>(o_mine, rescale ? alpha : 1.f);
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                ptx::mbar_arrive(&p_full[2 * sb + half]);
                ++gtile;
            }
            // ---------------------------------------------------------------- epilogue
            // Merge the two halves: exchange (m, l) with the partner warp of this quarter.
            xch[half * kBlockM + row] = m;
            xch[(2 + half) * kBlockM + row] = l;
            ptx::named_barrier_sync(pair_bar, 64);
            const float m_o = xch[(1 - half) * kBlockM + row];
            const float l_o = xch[(3 - half) * kBlockM + row];
            ptx::named_barrier_sync(pair_bar, 64);  // partner done reading before the next write
            const float m_a = half == 0 ? m : m_o, l_a = half == 0 ? l : l_o;
            const float m_b = half == 0 ? m_o : m, l_b = half == 0 ? l_o : l;
            const float mx = fmaxf(m_a, m_b);
            const float w_a = (l_a > 0.f) ? ptx::ex2(m_a - mx) : 0.f;
            const float w_b = (l_b > 0.f) ? ptx::ex2(m_b - mx) : 0.f;
            const float l_tot = l_a * w_a + l_b * w_b;
            const float inv_l = (l_tot > 0.f) ? 1.f / l_tot : 0.f;
            const float lse_val = (l_tot > 0.f) ? (mx + __log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
            // Both chains' last P.V must have landed (this thread reads its columns of both).
            wait_bar_warp(&pv_done[0], (gtile - 1) & 1, abort_flag, p.err);
            wait_bar_warp(&pv_done[1], (gtile - 1) & 1, abort_flag, p.err);
            ptx::tc_fence_after();

            constexpr int CW = DH < 32 ? DH : 32;   // columns merged per step
            __nv_bfloat16* outp = reinterpret_cast<__nv_bfloat16*>(p.out);
            const int Tu = p.tiles_per_unit;
            const bool whole = (MODE != kDecoderSample) || (it.t_begin == 0 && it.t_end == Tu);
            float* slot = nullptr;
            int c_first = 0, c_last = 0;
            long long ubeg = 0;
            if (MODE == kDecoderSample && !whole) {
                ubeg = static_cast<long long>(it.q_z) * Tu;
                c_first = owner_cta(ubeg, p.total_tiles, gridDim.x);
                c_last = owner_cta(ubeg + Tu - 1, p.total_tiles, gridDim.x);
                const int my_slot = (range_begin(blockIdx.x, p.total_tiles, gridDim.x) >= ubeg) ? 2 * blockIdx.x
                                                                                                : 2 * blockIdx.x + 1;
                slot = p.ws_partial + static_cast<size_t>(my_slot) * p.slot_floats;
            }
            uint8_t* stage = smem + SM::OFF_O;
            if (SM::STAGE_O) {
                if (stid == 0) ptx::tma_store_wait_read_all();
                ptx::named_barrier_sync(1, kSoftmaxThreads);
            }
#pragma unroll
            for (int c0 = 0; c0 < DH; c0 += CW) {
                float oa[CW], obv[CW], o[CW];
                load_tmem_cols<CW>(o_base + half * DH + c0, oa);
                load_tmem_cols<CW>(o_base + D + half * DH + c0, obv);
#pragma unroll
                for (int c = 0; c < CW; ++c)
                    o[c] = (w_a > 0.f ? oa[c] * w_a : 0.f) + (w_b > 0.f ? obv[c] * w_b : 0.f);
                const int col = half * DH + c0;  // first output column of this step
                if (SM::STAGE_O) {
                    // bf16 tile in the swizzled layout of the output tensor map
#pragma unroll
                    for (int g = 0; g < CW / 8; ++g) {
                        const int unit = (col + 8 * g) / 8;
                        const int ch = unit / (C::RB / 16);
                        const int u = unit % (C::RB / 16);
                        *reinterpret_cast<uint4*>(stage + ch * C::CHUNK_BYTES + swz_offset<C::RB>(row, u)) =
                            pack8_bf16(&o[8 * g], inv_l);
                    }
                } else if (MODE != kDecoderSample || whole) {
                    if (row_valid) {
                        const size_t r = (MODE == kDecoderSample)
                                             ? static_cast<size_t>(it.out_row0 + row)
                                             : static_cast<size_t>(it.q_z) * p.L + it.q_row0 + row;
                        uint4* dst = reinterpret_cast<uint4*>(outp + r * D + col);
#pragma unroll
                        for (int c = 0; c < CW; c += 8) dst[c / 8] = pack8_bf16(&o[c], inv_l);
                    }
                } else if (row_valid && row < p.rows_cap) {
                    float4* so = reinterpret_cast<float4*>(slot + static_cast<size_t>(row) * D + col);
#pragma unroll
                    for (int c = 0; c < CW; c += 4) so[c / 4] = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&o_free[ob]);

            if (MODE != kDecoderSample) {
                if (SM::STAGE_O) {
                    ptx::fence_proxy_async_smem();
                    ptx::named_barrier_sync(1, kSoftmaxThreads);
                    if (stid == 0) {
                        for (int ch = 0; ch < C::NCH; ++ch)
                            ptx::tma_store_3d(&p.tm_o, stage + ch * C::CHUNK_BYTES, ch * (C::RB / 2),
                                              it.q_row0, it.q_z);
                        ptx::tma_store_commit();
                    }
                }
                if (p.lse != nullptr && row_valid && half == 0)
                    p.lse[static_cast<size_t>(it.q_z) * p.L + it.q_row0 + row] = lse_val;
            } else if (whole) {
                if (p.lse != nullptr && row_valid && half == 0) p.lse[it.out_row0 + row] = lse_val;
            } else {
                // Split unit: (O, m, l) of this CTA is in its slot; take a ticket; the last CTA of
                // the unit merges every slot.
                if (row_valid && row < p.rows_cap && half == 0) {
                    slot[p.rows_cap * D + row] = mx;
                    slot[p.rows_cap * D + p.rows_cap + row] = l_tot;
                }
                __threadfence();
                ptx::named_barrier_sync(1, kSoftmaxThreads);
                if (stid == 0) {
                    const int ticket = atomicAdd(&p.ws_tickets[c_first], 1);
                    const int last = (ticket == c_last - c_first) ? 1 : 0;
                    if (last) p.ws_tickets[c_first] = 0;
                    *bcast = last;
                }
                ptx::named_barrier_sync(1, kSoftmaxThreads);
                const int is_last = *bcast;
                ptx::named_barrier_sync(1, kSoftmaxThreads);
                if (is_last) {
                    __threadfence();
                    if (row_valid && row < p.rows_cap) {
                        const long long T = p.total_tiles;
                        const int grid = gridDim.x;
                        auto slot_ptr = [&](int c) -> const float* {
                            const int si = (range_begin(c, T, grid) >= ubeg) ? 2 * c : 2 * c + 1;
                            return p.ws_partial + static_cast<size_t>(si) * p.slot_floats;
                        };
                        float mmax = -INFINITY;
                        for (int c = c_first; c <= c_last; ++c)
                            mmax = fmaxf(mmax, __ldcg(slot_ptr(c) + p.rows_cap * D + row));
                        const float muse = (mmax == -INFINITY) ? 0.f : mmax;
                        float ltot = 0.f;
                        for (int c = c_first; c <= c_last; ++c) {
                            const float* sl = slot_ptr(c);
                            const float mw = __ldcg(sl + p.rows_cap * D + row);
                            if (mw != -INFINITY) ltot += ptx::ex2(mw - muse) * __ldcg(sl + p.rows_cap * D + p.rows_cap + row);
                        }
                        const float inv = (ltot > 0.f) ? 1.f / ltot : 0.f;
                        uint4* dst = reinterpret_cast<uint4*>(outp + static_cast<size_t>(it.out_row0 + row) * D + half * DH);
#pragma unroll 1
                        for (int c0 = 0; c0 < DH; c0 += CW) {
                            float acc[CW];
#pragma unroll
                            for (int c = 0; c < CW; ++c) acc[c] = 0.f;
                            for (int c = c_first; c <= c_last; ++c) {
                                const float* sl = slot_ptr(c);
                                const float mw = __ldcg(sl + p.rows_cap * D + row);
                                if (mw == -INFINITY) continue;
                                const float w = ptx::ex2(mw - muse);
                                const float4* so = reinterpret_cast<const float4*>(sl + static_cast<size_t>(row) * D + half * DH + c0);
#pragma unroll
                                for (int c4 = 0; c4 < CW / 4; ++c4) {
                                    const float4 v = __ldcg(so + c4);
                                    acc[4 * c4 + 0] += w * v.x;
                                    acc[4 * c4 + 1] += w * v.y;
                                    acc[4 * c4 + 2] += w * v.z;
                                    acc[4 * c4 + 3] += w * v.w;
                                }
                            }
#pragma unroll
                            for (int c = 0; c < CW; c += 8) dst[(c0 + c) / 8] = pack8_bf16(&acc[c], inv);
                        }
                        if (p.lse != nullptr && half == 0)
                            p.lse[it.out_row0 + row] =
                                (ltot > 0.f) ? (mmax + __log2f(ltot)) * 0.69314718055994531f : -INFINITY;
                    }
                }
            }
            ++item_idx;
        }
        if (SM::STAGE_O && stid == 0) ptx::tma_store_wait_all();
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace e2d2
