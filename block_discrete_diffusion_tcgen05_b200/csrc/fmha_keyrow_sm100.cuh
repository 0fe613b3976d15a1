// fmha_keyrow_sm100.cuh -- the E2D2 sampling step with the keys on the tensor-memory lanes.
//
// A sampling call ("Encoder-Decoder Diffusion Language Models for Efficient Training and
// Inference", paper notes, sec. 3) attends the S noised queries of one block, for the G query
// heads that share a kv head, to the cached clean prefix and to their own block.  Per (batch,
// kv head) that is a short query side (G*S packed rows, 16..64 here) against a long key side.
// A 128-row query tile would leave most tensor-core rows (and most softmax threads) idle, so the
// two products are taken transposed:
//
//     S^T  = K Q^T      M = 128 keys (TMEM lanes),  N = packed query columns,  K = d
//     O^T += V^T P^T    M = d = 128 (TMEM lanes),   N = packed query columns,  K = keys
//
// The softmax of a key tile runs on 256 threads: thread = key (its TMEM lane), warpgroup = half
// of the query columns.  A query column's running max is shared by the 128 key threads of its
// warpgroup: each tile they vote whether any key beats it by more than 2^8 (log2 units); only
// then is the column max reduced across the warpgroup and the column of O^T rescaled.  The
// column sums stay per thread until the end of the unit.  P^T goes to shared memory (the B
// operand of the second product); K, V and Q arrive by TMA, K and V in separate rings so that a
// K stage is refilled as soon as its S^T product is done.
//
// The kernel is bound by HBM only if no key tile waits for a chain of hand-offs, so S^T (TMEM)
// and P^T (shared memory) are double-buffered and the two products have their own issuing warps:
// S^T of tile t+1 is computed while the softmax works on tile t, and O^T += V^T P^T of tile t is
// issued the moment its P^T is published.
//
// A unit's epilogue (normalise, or publish a partial and merge the partials of a split unit)
// would stall the key-tile pipeline for longer than the K/V rings can cover, so it runs on a
// warpgroup of its own: at the end of a unit the softmax warps only hand over their column sums
// (shared memory) and go on with the next unit, whose O^T lives in the other TMEM buffer.
//
// CTA = 16 warps: warp 0 loads Q and K, warp 1 owns tensor memory and issues S^T = K Q^T, warp 2
// loads V, warp 3 issues O^T += V^T P^T, warps 4..11 are the two softmax warpgroups, warps
// 12..15 the epilogue warpgroup (which, in an encoder block step, first copies the block's K/V
// into the cache for the units whose own-block tile it takes).  The work split over CTAs (units
// that fill whole rounds of the grid taken whole, last; the rest split stream-K over their key
// tiles, the last CTA to finish a unit merging the partials in CTA order) and the partial-slot
// format are those of the generic sampling kernel in fmha_sm100.cuh.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "fmha_sm100.cuh"
#include "ptx_sm100.cuh"

namespace e2d2 {

constexpr int kKrThreads = 512;         // 16 warps = 4 warpgroups
constexpr int kKrRegsControl = 64;      // warpgroup 0: TMA producers and MMA issuers
constexpr int kKrRegsSoftmax = 160;     // warpgroups 1, 2
constexpr int kKrRegsEpilogue = 120;    // warpgroup 3
static_assert(128 * kKrRegsControl + 256 * kKrRegsSoftmax + 128 * kKrRegsEpilogue <= 65536, "register split");

// N: packed query columns per unit, G*S rounded up to 16, 32 or 64.  Head dim 128.
template <int N>
struct KrCfg {
    static_assert(N == 16 || N == 32 || N == 64, "packed query columns");
    static constexpr int D = 128;
    static constexpr int NH = N / 2;                              // columns per softmax warpgroup
    static constexpr int PRB = 2 * N;                             // bytes per P^T row (one key)
    static constexpr uint32_t PSWZ = PRB == 128 ? 2u : (PRB == 64 ? 4u : 6u);  // 128/64/32-byte swizzle
    static constexpr int QCHUNK = N * 128;                        // Q: one 64-column chunk of N rows
    static constexpr int Q_BYTES = 2 * QCHUNK;
    static constexpr int KV_CHUNK = kBlockN * 128;                // K/V: one 64-column chunk of 128 keys
    static constexpr int KV_BYTES = 2 * KV_CHUNK;
    static constexpr int P_BYTES = kBlockN * PRB;
    // Ring stages (shared memory: QB Q + 2 P^T + NK K + NV V tiles + the epilogue staging within
    // 227 KB).  A V stage is held from its load until the P.V of its tile has run (after the
    // softmax), so the V ring bounds how far the loads run ahead: three stages.  At N = 64 that
    // takes Q single-buffered (the next unit's Q is loaded once the last S^T of the current one
    // has read it) and an 8 KB staging buffer.
    static constexpr int NK = 2;
    static constexpr int NV = 3;
    static constexpr int QB = (N == 64) ? 1 : 2;
    static constexpr int STG_BYTES = (N == 64) ? 8192 : 16384;
    // TMEM: S^T buffers at columns 0 and N, O^T buffers at 2N and 3N.
    static constexpr uint32_t TMEM_COLS = (4 * N <= 64) ? 64u : ((4 * N <= 128) ? 128u : 256u);
};

template <int N>
struct KrSmem {
    using C = KrCfg<N>;
    static constexpr int OFF_Q = 0;                               // [QB][2 chunks][N][128 B]
    static constexpr int OFF_P = OFF_Q + C::QB * C::Q_BYTES;      // [2][128 keys][PRB]
    static constexpr int OFF_K = OFF_P + 2 * C::P_BYTES;          // [NK][2 chunks][128][128 B]
    static constexpr int OFF_V = OFF_K + C::NK * C::KV_BYTES;     // [NV][2 chunks][128][128 B]
    static constexpr int OFF_STG = OFF_V + C::NV * C::KV_BYTES;   // epilogue staging
    static constexpr int STG_BYTES = C::STG_BYTES;
    static constexpr int OFF_BAR = OFF_STG + STG_BYTES;
    // q_full[2], q_empty[2], k_full[NK], k_empty[NK], v_full[NV], v_empty[NV], s_full[2],
    // s_free[2], p_full[2], pv_done[2], o_full[2], o_free[2], l_ready[2], l_free[2], qk_drain,
    // pv_drain, tmem_done, merge_full
    static constexpr int NBAR = 4 + 2 * C::NK + 2 * C::NV + 16 + 4;
    static constexpr int OFF_VOTE = ((OFF_BAR + NBAR * 8 + 15) / 16) * 16;  // u32 [2 wg][2 parity][4 warps]
    static constexpr int OFF_CMAX = OFF_VOTE + 2 * 2 * 4 * 4;     // float [2 wg][2 parity][4 warps][NH]
    static constexpr int OFF_LRED = OFF_CMAX + 2 * 2 * 4 * C::NH * 4;  // float [2 ob][2 wg][4 warps][NH]
    static constexpr int OFF_MROW = OFF_LRED + 2 * 2 * 4 * C::NH * 4;  // float [2 ob][N]
    static constexpr int OFF_MISC = OFF_MROW + 2 * N * 4;
    // + per-column scale of the epilogue [2][N], then the ragged prefix table (+ 8 scan sums)
    static constexpr int OFF_RG = ((OFF_MISC + 64 + 2 * N * 4 + 15) / 16) * 16;
    static constexpr int BYTES = OFF_RG + (kRaggedMaxBatch + 1 + 8) * 4;
    static constexpr int ALLOC = ((BYTES + 1023) / 1024) * 1024 + 1024;  // + alignment slack
};

// Position (in 16-byte chunks) of chunk c of a partial-slot column row of 128 floats: inside each
// quarter of the row (eight chunks) the chunk index is XORed with the quarter and the column's
// parity, so the eight threads of a merge quarter-warp (two columns x four quarters) read eight
// different bank groups.  A warp's publish of 32 consecutive values still covers one 128-byte
// segment.
__device__ __forceinline__ int slot_chunk(int c, int col) {
    return (c & ~7) | ((c & 7) ^ ((c >> 3) & 3) ^ ((col & 1) << 2));
}

// Reduces v[0..NH) over the 32 lanes of the warp with `op`, halving the columns a lane keeps at
// each exchange (NH/2 + NH/4 + ... shuffles instead of 5 per column).  Returns the result for
// column lane / (32 / NH); v is clobbered.
template <int NH, class Op>
__device__ __forceinline__ float warp_columns_reduce(float (&v)[NH], int lane, Op op) {
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int o = 16 >> step;
        const int width = NH >> step;
        if (width > 1) {
            const int half = width / 2;
            const bool upper = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < half; ++i) {
                const float send = upper ? v[i] : v[i + half];
                const float keep = upper ? v[i + half] : v[i];
                v[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, o));
            }
        } else {
            v[0] = op(v[0], __shfl_xor_sync(0xffffffffu, v[0], o));
        }
    }
    return v[0];
}

template <int NC>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[NC]) {
    static_assert(NC == 8 || NC == 16 || NC == 32, "columns per load");
    if constexpr (NC == 8) {
        ptx::tmem_ld8(taddr, r);
    } else if constexpr (NC == 16) {
        ptx::tmem_ld16(taddr, r);
    } else {
        ptx::tmem_ld32(taddr, r);
    }
}

// Byte offset of 16-byte unit `u` of row `r` in a swizzled tile with RB-byte rows (32/64/128-byte
// swizzle: bits 4.. of the address XOR bits 7..).
template <int RB>
__device__ __forceinline__ uint32_t swz_rows(int r, int u) {
    const uint32_t a = static_cast<uint32_t>(r * RB + u * 16);
    constexpr uint32_t mask = RB / 16 - 1;
    return a ^ (((a >> 7) & mask) << 4);
}

template <int N>
__global__ void __launch_bounds__(kKrThreads, 1) fmha_keyrow_kernel(const __grid_constant__ FmhaParams p) {
    using C = KrCfg<N>;
    using SM = KrSmem<N>;
    constexpr int NH = C::NH;
    constexpr int D = C::D;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    ptx::griddep_launch_dependents();  // the next kernel may launch; it waits for this one's end
#define E2D2_KR_POINTERS                                                                              \
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &       \
                                               ~static_cast<uintptr_t>(1023));                        \
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::OFF_BAR);                                 \
    uint64_t* q_full = bars;                                                                          \
    uint64_t* q_empty = q_full + 2;                                                                   \
    uint64_t* k_full = q_empty + 2;                                                                   \
    uint64_t* k_empty = k_full + C::NK;                                                               \
    uint64_t* v_full = k_empty + C::NK;                                                               \
    uint64_t* v_empty = v_full + C::NV;                                                               \
    uint64_t* s_full = v_empty + C::NV;     /* [2] S^T buffer written      */                        \
    uint64_t* s_free = s_full + 2;          /* [2] S^T buffer read         */                        \
    uint64_t* p_full = s_free + 2;          /* [2] P^T buffer written      */                        \
    uint64_t* pv_done = p_full + 2;         /* [2] P^T buffer consumed     */                        \
    uint64_t* o_full = pv_done + 2;         /* [2] O^T buffer complete     */                        \
    uint64_t* o_free = o_full + 2;          /* [2] O^T buffer read         */                        \
    uint64_t* l_ready = o_free + 2;         /* [2] unit column stats written */                      \
    uint64_t* l_free = l_ready + 2;         /* [2] unit column stats read    */                      \
    uint64_t* qk_drain = l_free + 2;                                                                  \
    uint64_t* pv_drain = qk_drain + 1;                                                                \
    uint64_t* tmem_done = pv_drain + 1;     /* softmax and epilogue threads are done with TMEM */    \
    uint64_t* merge_full = tmem_done + 1;   /* partial slots copied in for the final merge */        \
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SM::OFF_MISC);                         \
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM::OFF_MISC + 8);              \
    volatile int* bcast = reinterpret_cast<volatile int*>(smem + SM::OFF_MISC + 16);                  \
    int* rg_pre = reinterpret_cast<int*>(smem + SM::OFF_RG);                                          \
    (void)rg_pre;                                                                                     \
    (void)q_full; (void)q_empty; (void)k_full; (void)k_empty; (void)v_full; (void)v_empty;            \
    (void)s_full; (void)s_free; (void)p_full; (void)pv_done; (void)o_full; (void)o_free;              \
    (void)l_ready; (void)l_free; (void)qk_drain; (void)pv_drain; (void)tmem_done; (void)merge_full;   \
    (void)tmem_holder; (void)abort_flag; (void)bcast;
    uint32_t tmem_base;
    {
    E2D2_KR_POINTERS
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&q_full[i], 1);
            ptx::mbar_init(&q_empty[i], 1);
            ptx::mbar_init(&s_full[i], 1);
            ptx::mbar_init(&s_free[i], kSoftmaxThreads);
            ptx::mbar_init(&p_full[i], kSoftmaxThreads);
            ptx::mbar_init(&pv_done[i], 1);
            ptx::mbar_init(&o_full[i], 1);
            ptx::mbar_init(&o_free[i], 128);
            ptx::mbar_init(&l_ready[i], kSoftmaxThreads);
            ptx::mbar_init(&l_free[i], 128);
        }
        for (int i = 0; i < C::NK; ++i) {
            ptx::mbar_init(&k_full[i], 1);
            ptx::mbar_init(&k_empty[i], 1);
        }
        for (int i = 0; i < C::NV; ++i) {
            ptx::mbar_init(&v_full[i], 1);
            ptx::mbar_init(&v_empty[i], 1);
        }
        ptx::mbar_init(qk_drain, 1);
        ptx::mbar_init(pv_drain, 1);
        ptx::mbar_init(tmem_done, kSoftmaxThreads + 128);
        ptx::mbar_init(merge_full, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_holder, C::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::griddep_wait();  // inputs are read after the previous kernel on the stream has finished
    if (p.P_dev != nullptr) ragged_prefix(p, rg_pre, rg_pre + kRaggedMaxBatch + 1);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    tmem_base = *tmem_holder;
    }

    if (warp == 0 || warp == 2) {
        ptx::setmaxnreg_dec<kKrRegsControl>();
        E2D2_KR_POINTERS
        // -------------------------------------------------------------- TMA producers
        // Warp 0: Q (once per unit) and the K ring; warp 2: the V ring.  Both walk the schedule.
        const bool is_k = (warp == 0);
        const bool leader = ptx::elect_one();
        if (leader) {
            if (is_k) {
                ptx::tma_prefetch_desc(&p.tm_q);
                ptx::tma_prefetch_desc(&p.tm_k0);
                ptx::tma_prefetch_desc(&p.tm_k1);
            } else {
                ptx::tma_prefetch_desc(&p.tm_v0);
                ptx::tma_prefetch_desc(&p.tm_v1);
            }
        }
        __syncwarp();
        test_producer_delay();
        const int NS = is_k ? C::NK : C::NV;
        uint64_t* full = is_k ? k_full : v_full;
        uint64_t* empty = is_k ? k_empty : v_empty;
        const uint32_t ring_off = is_k ? SM::OFF_K : SM::OFF_V;
        Scheduler<kDecoderSample> sched(p, rg_pre);
        Item it;
        uint32_t iter = 0, item_idx = 0;
        bool ok = true;
        while (ok && sched.next(it)) {
            if (is_k) {
                const int qb = item_idx % C::QB;
                ok = wait_bar_warp(&q_empty[qb], ((item_idx / C::QB) & 1) ^ 1, abort_flag, p.err);
                if (!ok) break;
                if (leader) {
                    ptx::mbar_arrive_expect_tx(&q_full[qb], C::Q_BYTES);
                    for (int ch = 0; ch < 2; ++ch)
                        ptx::tma_load_2d(&p.tm_q, &q_full[qb], smem + SM::OFF_Q + qb * C::Q_BYTES + ch * C::QCHUNK,
                                         ch * 64, it.q_y);
                }
                __syncwarp();
            }
            ++item_idx;
            for (int t = it.t_begin; t < it.t_end; ++t) {
                const int st = iter % NS;
                ok = wait_bar_warp(&empty[st], ((iter / NS) & 1) ^ 1, abort_flag, p.err);
                // The first V loads wait for the first K tile: at launch every CTA asks for its
                // tiles at once, and Q + K0 (the first product's operands) land sooner without
                // three V tiles competing for the same DRAM bandwidth.
                if (ok && !is_k && iter == 0) ok = wait_bar_warp(&k_full[0], 0, abort_flag, p.err);
                if (!ok) break;
                const TileRef tr = tile_of<kDecoderSample>(p, it, t);
                // debug builds: the tile starts inside its source and the kv unit exists
                E2D2_DCHECK(tr.kt * kBlockN < (tr.src ? p.S : it.P), p.err);
                E2D2_DCHECK(it.kv_z >= 0 && it.kv_z < p.batch * p.kv_heads, p.err);
                if (leader) {
                    const CUtensorMap* m = is_k ? (tr.src ? &p.tm_k1 : &p.tm_k0) : (tr.src ? &p.tm_v1 : &p.tm_v0);
                    ptx::mbar_arrive_expect_tx(&full[st], static_cast<uint32_t>(tr.box_rows) * D * 2);
                    for (int ch = 0; ch < 2; ++ch)
                        ptx::tma_load_3d(m, &full[st], smem + ring_off + st * C::KV_BYTES + ch * C::KV_CHUNK, ch * 64,
                                         tr.kt * kBlockN, it.kv_z);
                }
                __syncwarp();
                ++iter;
            }
        }
        // Never leave with copies in flight.
        volatile int no_abort = 0;
        for (uint32_t i = iter > static_cast<uint32_t>(NS) ? iter - NS : 0u; i < iter; ++i)
            wait_bar_warp(&full[i % NS], (i / NS) & 1u, &no_abort, p.err, true);
        if (is_k)
            for (uint32_t i = item_idx > static_cast<uint32_t>(C::QB) ? item_idx - C::QB : 0u; i < item_idx; ++i)
                wait_bar_warp(&q_full[i % C::QB], (i / C::QB) & 1u, &no_abort, p.err, true);
    } else if (warp == 1) {
        ptx::setmaxnreg_dec<kKrRegsControl>();
        E2D2_KR_POINTERS
        // -------------------------------------------------------------- S^T = K Q^T issuer
        const bool leader = ptx::elect_one();
        const uint32_t smem_base = ptx::smem_u32(smem);
        const uint32_t sQ = smem_base + SM::OFF_Q, sK = smem_base + SM::OFF_K;
        const uint64_t kdesc = ptx::smem_desc(0, 16, 1024, 2u);  // K (A) and Q (B): K-major, 128B swizzle
        constexpr uint32_t idesc_s = ptx::idesc_bf16_f32(kBlockN, N, false, false);
        Scheduler<kDecoderSample> sched(p, rg_pre);
        Item it;
        uint32_t kit = 0, item_idx = 0, tc = 0;
        bool ok = true;
        while (ok && sched.next(it)) {
            const uint32_t qb = item_idx % C::QB;
            ok = wait_bar_warp(&q_full[qb], (item_idx / C::QB) & 1, abort_flag, p.err);
            for (int t = it.t_begin; t < it.t_end && ok; ++t) {
                const uint32_t sb = tc & 1;
                const uint32_t kst = kit % C::NK;
                ok = wait_bar_warp(&s_free[sb], ((tc >> 1) & 1) ^ 1, abort_flag, p.err) &&
                     wait_bar_warp(&k_full[kst], (kit / C::NK) & 1, abort_flag, p.err);
                if (!ok) break;
                ptx::tc_fence_after();
                if (leader) {
                    const uint32_t k_base = sK + kst * C::KV_BYTES;
                    const uint32_t q_base = sQ + qb * C::Q_BYTES;
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t ka = k_base + (ks / 4) * C::KV_CHUNK + (ks % 4) * 32;
                        const uint32_t qa = q_base + (ks / 4) * C::QCHUNK + (ks % 4) * 32;
                        ptx::mma_ss(tmem_base + sb * N, kdesc | (ka >> 4), kdesc | (qa >> 4), idesc_s, ks > 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(&k_empty[kst]);
                    ptx::mma_commit(&s_full[sb]);
                    if (t == it.t_end - 1) ptx::mma_commit(&q_empty[qb]);
                }
                __syncwarp();
                ++kit;
                ++tc;
            }
            ++item_idx;
        }
        // Drain: this warp's products, the other issuer's, and every softmax and epilogue thread
        // are done with tensor memory before it is released.
        if (leader) ptx::mma_commit(qk_drain);
        __syncwarp();
        volatile int no_abort = 0;
        wait_bar_warp(qk_drain, 0, &no_abort, p.err, true);
        wait_bar_warp(pv_drain, 0, &no_abort, p.err, true);
        wait_bar_warp(tmem_done, 0, &no_abort, p.err, true);
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, C::TMEM_COLS);
    } else if (warp == 3) {
        ptx::setmaxnreg_dec<kKrRegsControl>();
        E2D2_KR_POINTERS
        // -------------------------------------------------------------- O^T += V^T P^T issuer
        const bool leader = ptx::elect_one();
        const uint32_t smem_base = ptx::smem_u32(smem);
        const uint32_t sP = smem_base + SM::OFF_P, sV = smem_base + SM::OFF_V;
        const uint64_t vdesc = ptx::smem_desc(0, C::KV_CHUNK, 1024, 2u);             // V^T: MN-major (d contiguous)
        const uint64_t pdesc = ptx::smem_desc(0, C::P_BYTES, 8 * C::PRB, C::PSWZ);    // P^T: MN-major
        constexpr uint32_t idesc_o = ptx::idesc_bf16_f32(D, N, true, true);
        Scheduler<kDecoderSample> sched(p, rg_pre);
        Item it;
        uint32_t vit = 0, item_idx = 0, tc = 0;
        bool ok = true;
        while (ok && sched.next(it)) {
            const uint32_t ob = item_idx & 1;
            for (int t = it.t_begin; t < it.t_end && ok; ++t) {
                const uint32_t sb = tc & 1;
                const uint32_t vst = vit % C::NV;
                const bool first = (t == it.t_begin);
                ok = wait_bar_warp(&p_full[sb], (tc >> 1) & 1, abort_flag, p.err) &&
                     (!first || wait_bar_warp(&o_free[ob], ((item_idx >> 1) & 1) ^ 1, abort_flag, p.err)) &&
                     wait_bar_warp(&v_full[vst], (vit / C::NV) & 1, abort_flag, p.err);
                if (!ok) break;
                ptx::tc_fence_after();
                const TileRef tr = tile_of<kDecoderSample>(p, it, t);
                if (leader) {
                    const uint32_t d_tmem = tmem_base + 2 * N + ob * N;
                    const uint32_t v_base = sV + vst * C::KV_BYTES;
                    const uint32_t p_base = sP + sb * C::P_BYTES;
                    for (int ks = 0; ks < tr.nk16 / 16; ++ks)
                        ptx::mma_ss(d_tmem, vdesc | ((v_base + ks * 16 * 128) >> 4),
                                    pdesc | ((p_base + ks * 16 * C::PRB) >> 4), idesc_o, (first && ks == 0) ? 0u : 1u);
                    ptx::mma_commit(&v_empty[vst]);
                    ptx::mma_commit(&pv_done[sb]);
                    if (t == it.t_end - 1) ptx::mma_commit(&o_full[ob]);
                }
                __syncwarp();
                ++vit;
                ++tc;
            }
            ++item_idx;
        }
        if (leader) ptx::mma_commit(pv_drain);
        __syncwarp();
    } else if (warp < 12) {
        ptx::setmaxnreg_inc<kKrRegsSoftmax>();
        E2D2_KR_POINTERS
        // -------------------------------------------------------------- softmax warpgroups
        // Thread = key lane 32*w + lane of S^T; warpgroup g owns query columns [g*NH, g*NH + NH).
        // Waits never break the loops: every warp takes every named barrier.
        const int g = (warp - 4) >> 2;
        const int w = warp & 3;
        const int key = 32 * w + lane;
        const int colbase = g * NH;
        const uint32_t lane_off = static_cast<uint32_t>(32 * w) << 16;
        const uint32_t wg_bar = 1 + g;
        const float sl2 = p.scale_log2;
        const int rows = p.rows_per_unit;
        uint32_t* vote = reinterpret_cast<uint32_t*>(smem + SM::OFF_VOTE) + g * 8;
        float* cmax = reinterpret_cast<float*>(smem + SM::OFF_CMAX) + g * 2 * 4 * NH;
        uint8_t* sP = smem + SM::OFF_P;
        Scheduler<kDecoderSample> sched(p, rg_pre);
        Item it;
        uint32_t tc = 0, item_idx = 0;
        while (sched.next(it)) {
            const uint32_t ob = item_idx & 1;
            float m_run[NH], l_part[NH];
#pragma unroll
            for (int j = 0; j < NH; ++j) {
                m_run[j] = -INFINITY;
                l_part[j] = 0.f;
            }
            for (int t = it.t_begin; t < it.t_end; ++t) {
                // Tile tc uses S^T / P^T buffer sb; phases of each buffer's barriers count its uses.
                const uint32_t sb = tc & 1, use = tc >> 1;
                wait_bar_warp(&s_full[sb], use & 1, abort_flag, p.err);
                ptx::tc_fence_after();
                const TileRef tr = tile_of<kDecoderSample>(p, it, t);
                const int len = tr.src ? p.S : it.P;
                const bool key_ok = key < min(kBlockN, len - tr.kt * kBlockN);
                float x[NH];
                {
                    uint32_t raw[NH];
                    tmem_ld_cols<NH>(tmem_base + sb * N + lane_off + colbase, raw);
                    ptx::tmem_wait_ld();
                    ptx::reg_fence<NH>(raw);
#pragma unroll
                    for (int j = 0; j < NH; ++j)
                        x[j] = (key_ok && colbase + j < rows) ? __uint_as_float(raw[j]) * sl2 : -INFINITY;
                }
                ptx::tc_fence_before();
                ptx::mbar_arrive(&s_free[sb]);  // the next S^T product may overwrite the buffer
                // Vote: does any key of the tile beat a column's running max by more than 2^8?
                uint32_t e = 0;
#pragma unroll
                for (int j = 0; j < NH; ++j) e |= (x[j] > m_run[j] + kRescaleThreshold) ? (1u << j) : 0u;
                e = __reduce_or_sync(0xffffffffu, e);
                const uint32_t par = tc & 1;
                if (lane == 0) vote[par * 4 + w] = e;
                ptx::named_barrier_sync(wg_bar, 128);
                const uint4 vv = *reinterpret_cast<const uint4*>(vote + par * 4);
                const uint32_t E = vv.x | vv.y | vv.z | vv.w;
                if (E != 0) {
                    // New maxima: reduce the voted columns over the 128 keys of the warpgroup.
                    float tmp[NH];
#pragma unroll
                    for (int j = 0; j < NH; ++j) tmp[j] = x[j];
                    const float mine = warp_columns_reduce<NH>(tmp, lane, [](float a, float b) { return fmaxf(a, b); });
                    float* cm = cmax + par * 4 * NH;
                    if ((lane % (32 / NH)) == 0) cm[w * NH + lane / (32 / NH)] = mine;
                    ptx::named_barrier_sync(wg_bar, 128);
                    const bool rescale_o = (t != it.t_begin);
                    const uint32_t o_tmem = tmem_base + lane_off + 2 * N + ob * N + colbase;
                    if (rescale_o) {
                        // O^T holds every product up to tile tc-1 only once that one has landed.
                        wait_bar_warp(&pv_done[sb ^ 1], ((tc - 1) >> 1) & 1, abort_flag, p.err);
                        ptx::tc_fence_after();
                    }
                    // Eight columns at a time, each group one branch-free block (per-column branches
                    // made each column a dependent chain of its own): the new max where the vote moved
                    // it, the factor 2^(m_old - m_new) (0 for a column's first keys, 1 where nothing
                    // moved), then the group's O^T columns if any of them moved.
#pragma unroll
                    for (int c0 = 0; c0 < NH; c0 += 8) {
                        float fac[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int j = c0 + i;
                            const float tm = fmaxf(fmaxf(cm[j], cm[NH + j]), fmaxf(cm[2 * NH + j], cm[3 * NH + j]));
                            const float mn = ((E >> j) & 1u) ? tm : m_run[j];
                            fac[i] = ptx::ex2(mn == m_run[j] ? 0.f : m_run[j] - mn);
                            m_run[j] = mn;
                            l_part[j] *= fac[i];
                        }
                        if (rescale_o && ((E >> c0) & 0xffu) != 0) {
                            uint32_t o[8];
                            ptx::tmem_ld8(o_tmem + c0, o);
                            ptx::tmem_wait_ld();
                            ptx::reg_fence<8>(o);
#pragma unroll
                            for (int i = 0; i < 8; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * fac[i]);
                            ptx::tmem_st8(o_tmem + c0, o);
                        }
                    }
                    if (rescale_o) ptx::tmem_wait_st();
                }
                // P^T row of this key: exp2(x - m), packed to bf16, into the swizzled B tile.
                uint32_t pk[NH / 2];
#pragma unroll
                for (int j = 0; j < NH; j += 2) {
                    const float e0 = (colbase + j < rows) ? ptx::ex2(x[j] - m_run[j]) : 0.f;
                    const float e1 = (colbase + j + 1 < rows) ? ptx::ex2(x[j + 1] - m_run[j + 1]) : 0.f;
                    l_part[j] += e0;
                    l_part[j + 1] += e1;
                    pk[j / 2] = ptx::pack_bf16x2(e0, e1);
                }
                // P^T buffer sb was last read by the product of tile tc-2.
                wait_bar_warp(&pv_done[sb], (use & 1) ^ 1, abort_flag, p.err);
                uint8_t* pbuf = sP + sb * C::P_BYTES;
#pragma unroll
                for (int u = 0; u < NH / 8; ++u)
                    *reinterpret_cast<uint4*>(pbuf + swz_rows<C::PRB>(key, colbase / 8 + u)) =
                        make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
                if (g == 0 && p.P_dev != nullptr && tr.src == 0 && it.P - tr.kt * kBlockN < tr.nk16) {
                    // Ragged prefix: cache rows at or past P[b] in this tile may hold anything (NaN
                    // included) and O^T += V^T P^T would meet them with p = 0; zero those V rows.
                    const uint32_t vst = tc % C::NV;
                    wait_bar_warp(&v_full[vst], (tc / C::NV) & 1u, abort_flag, p.err);
                    if (key >= it.P - tr.kt * kBlockN && key < tr.nk16) {
#pragma unroll
                        for (int ch = 0; ch < 2; ++ch) {
                            uint4* dst = reinterpret_cast<uint4*>(smem + SM::OFF_V + vst * C::KV_BYTES + ch * C::KV_CHUNK +
                                                                  key * 128);
#pragma unroll
                            for (int u = 0; u < 8; ++u) dst[u] = make_uint4(0u, 0u, 0u, 0u);
                        }
                    }
                }
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                ptx::mbar_arrive(&p_full[sb]);
                ++tc;
            }
            // Hand the unit's column statistics to the epilogue warpgroup: per column the running
            // max (identical in every thread) and the sum over this warpgroup's 128 keys.
            wait_bar_warp(&l_free[ob], ((item_idx >> 1) & 1) ^ 1, abort_flag, p.err);
            {
                float* lred = reinterpret_cast<float*>(smem + SM::OFF_LRED) + (ob * 2 + g) * 4 * NH;
                const float mine = warp_columns_reduce<NH>(l_part, lane, [](float a, float b) { return a + b; });
                if ((lane % (32 / NH)) == 0) lred[w * NH + lane / (32 / NH)] = mine;
                if (w == 0) {
                    float mv = 0.f;
#pragma unroll
                    for (int j = 0; j < NH; ++j) mv = (lane == j) ? m_run[j] : mv;
                    if (lane < NH) reinterpret_cast<float*>(smem + SM::OFF_MROW)[ob * N + colbase + lane] = mv;
                }
            }
            ptx::mbar_arrive(&l_ready[ob]);
            ++item_idx;
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(tmem_done);
    } else {
        ptx::setmaxnreg_dec<kKrRegsEpilogue>();
        E2D2_KR_POINTERS
        // -------------------------------------------------------------- epilogue warpgroup
        // Thread = head-dim row d = 32*w + lane of O^T (its TMEM lane); all N columns, EG at a time.
        const int w = warp & 3;
        const int d = 32 * w + lane;
        const int wtid = threadIdx.x - 384;
        const uint32_t lane_off = static_cast<uint32_t>(32 * w) << 16;
        const int rows = p.rows_per_unit;
        const int cap = p.rows_cap;
        __nv_bfloat16* outp = reinterpret_cast<__nv_bfloat16*>(p.out);
        const float* mrow_all = reinterpret_cast<const float*>(smem + SM::OFF_MROW);
        const float* lred_all = reinterpret_cast<const float*>(smem + SM::OFF_LRED);
        Scheduler<kDecoderSample> sched(p, rg_pre);
        Item it;
        uint32_t item_idx = 0;
        while (sched.next(it)) {
            const uint32_t ob = item_idx & 1;
            // Encoder block step: the unit's own block joins the cache (the CTA that takes the
            // own-block tile writes it, while its first products are still running).
            if (p.app_dst_k != nullptr && it.t_begin == 0) append_block_rows(p, D, it.kv_z, wtid, 128);
            wait_bar_warp(&o_full[ob], (item_idx >> 1) & 1, abort_flag, p.err);
            wait_bar_warp(&l_ready[ob], (item_idx >> 1) & 1, abort_flag, p.err);
            ptx::tc_fence_after();
            const int Tu = it.tu;
            const bool whole = (it.t_begin == 0 && it.t_end == Tu);
            const long long ubeg = it.ubeg;
            const long long T = it.total;
            const int grid = it.sgrid;
            const int c_first = whole ? 0 : owner_cta(ubeg, T, grid);
            const int c_last = whole ? 0 : owner_cta(ubeg + Tu - 1, T, grid);
            auto slot_of = [&](int c) -> float* {
                const int si = (range_begin(c, T, grid) >= ubeg) ? 2 * c : 2 * c + 1;
                return p.ws_partial + static_cast<size_t>(si) * p.slot_floats;
            };
            float* slot = whole ? nullptr : slot_of(blockIdx.x);
            const float* mrow = mrow_all + ob * N;
            // Per column, once: the normaliser (whole unit) and the LSE, or the slot's m and l.
            // (double-buffered by unit parity: a thread still scaling this unit's columns cannot
            // meet the next unit's writes, which come after the next unit's barrier)
            float* colscale = reinterpret_cast<float*>(smem + SM::OFF_MISC + 64) + ob * N;
            if (wtid < N) {
                const int col = wtid;
                const float* lr = lred_all + (ob * 2 + col / NH) * 4 * NH + col % NH;
                const float l = (lr[0] + lr[NH]) + (lr[2 * NH] + lr[3 * NH]);
                const float m = mrow[col];
                colscale[col] = (whole && l > 0.f) ? 1.f / l : 1.f;
                if (whole) {
                    if (p.lse != nullptr && col < rows)
                        p.lse[it.out_row0 + col] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
                } else if (col < cap) {
                    slot[cap * D + col] = m;
                    slot[cap * D + cap + col] = l;
                }
            }
            // O^T of the unit into registers (this thread's head-dim row, every column), then the
            // buffer is free for the next unit's products.
            constexpr int LW = N < 32 ? N : 32;  // columns per TMEM load
            uint32_t raw[N];
#pragma unroll
            for (int c0 = 0; c0 < N; c0 += LW) {
                const uint32_t ta = tmem_base + lane_off + 2 * N + ob * N + c0;
                if constexpr (LW == 32) ptx::tmem_ld32(ta, raw + c0);
                else ptx::tmem_ld16(ta, *reinterpret_cast<uint32_t(*)[16]>(raw + c0));
            }
            ptx::tmem_wait_ld();
            ptx::reg_fence<N>(raw);
            ptx::tc_fence_before();
            ptx::mbar_arrive(&o_free[ob]);
            if (wtid == 0) ptx::tma_store_wait_read_all();  // the last unit's output has left the staging buffer
            ptx::named_barrier_sync(3, 128);  // colscale written, column statistics read
            ptx::mbar_arrive(&l_free[ob]);
            // The unit's rows: a whole unit's bf16 output rows out_row0.. go through the staging
            // buffer; a split unit's fp32 [col][D] partial goes straight from registers to its slot
            // (for each column a warp writes 32 consecutive head-dim values, one 128-byte segment).
            if (whole) {
                // bf16 rows staged in shared memory (a pass of columns per staging buffer) and
                // written with one bulk copy per pass
                constexpr int PASS = SM::STG_BYTES / (D * 2);
                __nv_bfloat16* st = reinterpret_cast<__nv_bfloat16*>(smem + SM::OFF_STG) + d;
#pragma unroll
                for (int c_lo = 0; c_lo < N; c_lo += PASS) {
                    if (c_lo >= rows) break;
                    if (c_lo > 0) {
                        if (wtid == 0) ptx::tma_store_wait_read_all();  // the previous pass has been read
                        ptx::named_barrier_sync(3, 128);
                    }
#pragma unroll
                    for (int c = c_lo; c < c_lo + PASS && c < N; ++c)
                        st[(c - c_lo) * D] = __float2bfloat16_rn(__uint_as_float(raw[c]) * colscale[c]);
                    ptx::fence_proxy_async_smem();
                    ptx::named_barrier_sync(3, 128);
                    if (wtid == 0) {
                        const int c_hi = min(rows, c_lo + PASS);
                        ptx::bulk_store_s2g(outp + static_cast<size_t>(it.out_row0 + c_lo) * D,
                                            smem + SM::OFF_STG, static_cast<uint32_t>(c_hi - c_lo) * D * 2);
                        ptx::tma_store_commit();
                    }
                }
            } else {
                const int off0 = slot_chunk(d >> 2, 0) * 4 + (d & 3), off1 = slot_chunk(d >> 2, 1) * 4 + (d & 3);
#pragma unroll
                for (int c = 0; c < N; ++c)
                    if (c < cap) slot[static_cast<size_t>(c) * D + ((c & 1) ? off1 : off0)] = __uint_as_float(raw[c]);
            }
            if (!whole) {
                // Release: the barrier orders every thread's slot stores before one thread's fence
                // and ticket.  The last CTA of the unit gets ticket c_last - c_first.
                ptx::named_barrier_sync(3, 128);
                if (wtid == 0) {
                    __threadfence();
                    const int ticket = atomicAdd(&p.ws_tickets[c_first], 1);
                    const int last = (ticket == c_last - c_first) ? 1 : 0;
                    if (last) p.ws_tickets[c_first] = 0;
                    *bcast = last;
                }
                ptx::named_barrier_sync(3, 128);
                const int is_last = *bcast;
                ptx::named_barrier_sync(3, 128);
                // In the CTA's last unit every K/V, Q and P^T buffer is free (the producers are done
                // and every product of the unit has landed), and so is the staging buffer (an earlier
                // unit's output store finished reading it before this unit's first barrier): the
                // partial slots are then copied in with one bulk copy each, all in flight at once, and
                // merged from shared memory.
                const int nparts = c_last - c_first + 1;
                const uint32_t slot_bytes = static_cast<uint32_t>(p.slot_floats) * 4u;
                Scheduler<kDecoderSample> peek = sched;
                Item next_it;
                const bool in_smem = is_last && !peek.next(next_it) &&
                                     static_cast<uint32_t>(nparts) * slot_bytes <=
                                         static_cast<uint32_t>(SM::OFF_STG + SM::STG_BYTES - SM::OFF_Q);
                bool go = is_last;
                const uint8_t* region = smem + SM::OFF_Q;
                if (in_smem) {
                    __threadfence();
                    if (wtid == 0) {
                        ptx::fence_proxy_async_global();
                        ptx::mbar_arrive_expect_tx(merge_full, static_cast<uint32_t>(nparts) * slot_bytes);
                        for (int c = c_first; c <= c_last; ++c)
                            ptx::bulk_load_g2s(smem + SM::OFF_Q + (c - c_first) * slot_bytes, slot_of(c), slot_bytes,
                                               merge_full);
                    }
                    // If the copies never landed (bounded wait gave up: error word set), the
                    // slots are not merged and out / lse are left untouched.
                    go = wait_bar_warp(merge_full, 0, abort_flag, p.err);
                } else if (is_last) {
                    __threadfence();
                }
                // Online merge over the partials in CTA order (the result does not depend on which
                // CTA merges).  Thread = (column, 32 head-dim values): the eight 16-byte loads of one
                // partial are independent; the slot's chunk swizzle spreads the eight threads of a
                // quarter-warp over all 32 banks.
                const int q4 = wtid & 3;
                // One partial of the merge: m, l and this thread's 32 values of column col.
                auto merge_one = [&](float& mm, float& ll, float (&acc)[32], float mc, float lc, const float4 (&v)[8]) {
                    const float mn = fmaxf(mm, mc);
                    const float wa = (mm == -INFINITY) ? 0.f : ptx::ex2(mm - mn);
                    const float wb = (mc == -INFINITY) ? 0.f : ptx::ex2(mc - mn);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        acc[4 * i + 0] = acc[4 * i + 0] * wa + v[i].x * wb;
                        acc[4 * i + 1] = acc[4 * i + 1] * wa + v[i].y * wb;
                        acc[4 * i + 2] = acc[4 * i + 2] * wa + v[i].z * wb;
                        acc[4 * i + 3] = acc[4 * i + 3] * wa + v[i].w * wb;
                    }
                    ll = ll * wa + lc * wb;
                    mm = mn;
                };
#pragma unroll 1
                for (int col = wtid >> 2; go && col < cap; col += 32) {
                    float mm = -INFINITY, ll = 0.f, acc[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) acc[i] = 0.f;
                    const int sw = q4 ^ ((col & 1) << 2);
                    if (in_smem) {
#pragma unroll 1
                        for (int c = 0; c < nparts; ++c) {
                            const float* sl = reinterpret_cast<const float*>(region + c * slot_bytes);
                            const float4* row = reinterpret_cast<const float4*>(sl + col * D) + 8 * q4;
                            float4 v[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) v[i] = row[i ^ sw];
                            merge_one(mm, ll, acc, sl[cap * D + col], sl[cap * D + cap + col], v);
                        }
                    } else {
                        // two partials in flight
#pragma unroll 2
                        for (int c = 0; c < nparts; ++c) {
                            const float* sl = slot_of(c_first + c);
                            const float4* row =
                                reinterpret_cast<const float4*>(sl + static_cast<size_t>(col) * D) + 8 * q4;
                            float4 v[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) v[i] = __ldcg(row + (i ^ sw));
                            merge_one(mm, ll, acc, __ldcg(sl + cap * D + col), __ldcg(sl + cap * D + cap + col), v);
                        }
                    }
                    const float inv = ll > 0.f ? 1.f / ll : 0.f;
                    uint4* dst = reinterpret_cast<uint4*>(outp + static_cast<size_t>(it.out_row0 + col) * D + 32 * q4);
#pragma unroll
                    for (int i = 0; i < 4; ++i) dst[i] = pack8_bf16(&acc[8 * i], inv);
                    if (p.lse != nullptr && q4 == 0)
                        p.lse[it.out_row0 + col] = ll > 0.f ? (mm + __log2f(ll)) * 0.69314718055994531f : -INFINITY;
                }
            }
            ++item_idx;
        }
        if (wtid == 0) ptx::tma_store_wait_all();  // the staging buffer is read before the CTA exits
        ptx::tc_fence_before();
        ptx::mbar_arrive(tmem_done);
    }
#undef E2D2_KR_POINTERS
}

}  // namespace e2d2
