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
// CTA = 12 warps: warp 0 issues TMA loads, warp 1 owns tensor memory and issues tcgen05.mma,
// warps 2..3 write the block's K/V into the cache in an encoder block step (otherwise idle),
// warps 4..7 and 8..11 are two softmax warpgroups.  Per key tile of up to 128 keys:
//     S  = Q K^T          tcgen05.mma, A = Q (smem), B = K (smem, K-major)  -> TMEM (fp32)
//     P  = exp2(S*c - m)  softmax warpgroup, written back over S as bf16  -> TMEM
//     O += P V            tcgen05.mma, A = P (TMEM), B = V (smem, MN-major) -> TMEM
// Train calls take two 128-row query tiles per work item (one per softmax warpgroup) against
// one shared K/V stream.  At head_dim <= 64 the S of both query tiles rotate through three TMEM
// buffers (S number n in buffer n % 3): S(n) is issued as soon as P.V(n-3) has freed its buffer,
// so a warpgroup's next S is ready when it finishes the current P, and neither warpgroup waits
// for the tensor core; the P.V are issued in order as their P arrive, and at the end of an item
// all of them at once (the epilogue waits for the last).  At head_dim 128 (no TMEM for a third
// buffer) the MMA warp issues P.V(A, j-1), S(A, j), P.V(B, j-1), S(B, j), one S buffer per query
// tile.  The sampling call (shapes the
// keys-on-lanes kernel of fmha_keyrow_sm100.cuh does not take) uses one query tile holding all
// G*S packed rows of a kv head, with S double-buffered in TMEM instead.
// Each thread owns one query row (its TMEM lane) and all 128 key columns of a tile, read from
// TMEM in one pass.  A running max is only moved when it grows by more than 2^8 (log2 units), so
// O is rescaled rarely; the final normalisation uses the same max and is exact.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx_sm100.cuh"

namespace e2d2 {

enum Mode : int { kEncoder = 0, kDecoderTrain = 1, kDecoderSample = 2 };

constexpr int kBlockM = 128;            // query rows per tile (TMEM lanes)
constexpr int kBlockN = 128;            // keys per tile
constexpr int kThreads = 384;           // 12 warps = 3 warpgroups
constexpr int kSoftmaxThreads = 256;    // warpgroups 1 and 2 (warps 4..11)
// Register split (setmaxnreg): the launch gives every thread kRegsLaunch registers; warpgroup 0
// (TMA producer, MMA issuer, two mostly idle warps) gives most of its share to the softmax groups.
constexpr int kRegsLaunch = 168;
constexpr int kRegsControl = 88;
constexpr int kRegsSoftmax = 208;
static_assert(128 * kRegsControl + 256 * kRegsSoftmax <= kThreads * kRegsLaunch, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;
constexpr int kSampleMaxCtas = 256;     // upper bound of the sampling grid (workspace sizing)
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s per wait

// Bits of the device error word: a bounded wait gave up; a debug-build bounds check failed.
constexpr unsigned int kErrWaitTimeout = 1u;
constexpr unsigned int kErrDeviceCheck = 2u;

// Debug builds (E2D2_DEBUG): device-side bounds checks that record kErrDeviceCheck in the error
// word and carry on (TMA coordinates past a tensor's extent read zeros, so nothing faults).
#ifdef E2D2_DEBUG
#define E2D2_DCHECK(cond, err)                                  \
    do {                                                        \
        if (!(cond)) atomicOr((err), e2d2::kErrDeviceCheck);     \
    } while (0)
#else
#define E2D2_DCHECK(cond, err) \
    do {                       \
    } while (0)
#endif

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
    int num_qtiles;     // train: pairs of query tiles per head; sample: query tiles per (b, kv head)
    int rows_per_unit;  // sample: G * S packed query rows per (b, kv head)
    int tiles_per_unit; // sample: key tiles per unit
    long long total_tiles;  // sample: key tiles of the split units (split_units * tiles_per_unit)
    int split_units;    // sample: units split stream-K over CTAs [0, split_ctas), processed first
    int split_ctas;
    int whole_units;    // sample: units after the split ones, one CTA each, round robin
    int slot_floats;    // sample: floats per partial slot
    int rows_cap;       // sample: rows stored per partial slot
    int q_chunk;        // sample: packed query rows per TMEM lane quarter (multiple of 8, <= 32)
    // sample, encoder block step only (null otherwise): the block's K/V rows are also written to
    // the cache, rows P..P+S-1 of every (batch, kv head), by the CTA that takes the unit's own-block
    // tile.  Rows [0, P) are the only cache rows the attention reads, so the two never overlap.
    const uint4* app_src_k;  // [B*Hkv][S][D] bf16
    const uint4* app_src_v;
    uint4* app_dst_k;        // [B*Hkv][capacity][D] bf16
    uint4* app_dst_v;
    int app_capacity;
    // sample, ragged prefixes only (null otherwise): entry b's queries see cache rows [0, P_dev[b])
    // (clamped to [0, rg_capacity]); every unit's key tiles form one stream-K stream over all CTAs.
    const int* P_dev;
    int rg_capacity;
    int rg_units_per_entry;  // kv heads x query tiles per kv head
};

constexpr int kRaggedMaxBatch = 256;  // entries of a ragged sampling call (one per thread of the prefix scan)
constexpr int kMinRaggedTiles = 3;    // tiles per CTA the ragged split aims for
// P.V completions of a query tile go round a ring of this many barriers (P.V number j to barrier
// j % kPvRing).  A softmax warp waits for the previous P.V only when it rescales O; with one
// barrier, skipped waits could leave it two phases behind and a parity wait would pass early.
// When the softmax works on tile t, every P.V of that query tile up to t - 3 has completed (the
// S it reads was issued after them, and the tensor core runs in order) and P.V t + k cannot
// complete before tile t + k's P exists, so a ring of four keeps each wait unambiguous.
constexpr int kPvRing = 4;

// Train calls: an explicit order of the work items, computed on the host (longest processing
// time first: each item, longest first, goes to the CTA with the least work so far).  CTA c takes
// items item[first[c]] .. item[first[c + 1] - 1] in that order.  Without it (enabled = 0: more
// items or CTAs than the table holds) CTA c takes items c, c + grid, c + 2 grid, ...
constexpr int kOrderMaxCtas = 160;
constexpr int kOrderMaxItems = 1152;
struct ItemOrder {
    int enabled;
    uint16_t first[kOrderMaxCtas + 1];
    uint16_t item[kOrderMaxItems];
};
struct NoOrder {
    int enabled;
};
template <int MODE>
struct OrderOf {
    using type = ItemOrder;
};
template <>
struct OrderOf<kDecoderSample> {
    using type = NoOrder;
};

__host__ __device__ __forceinline__ int ragged_clamp(int P, int capacity) {
    return P < 0 ? 0 : (P > capacity ? capacity : P);
}

// Key tiles of one batch entry of a ragged sampling call: its units' own-block tiles and prefix
// tiles (128 keys each).
__host__ __device__ __forceinline__ int ragged_entry_tiles(int P, int S, int units_per_entry) {
    return units_per_entry * ((S + 127) / 128 + (P + 127) / 128);
}

// pre[b] = key tiles of entries 0..b-1 (pre[0] = 0, pre[batch] = all tiles), in shared memory.
// Every thread of the block calls it (one __syncthreads inside); threads 0..255 scan.
__device__ __forceinline__ void ragged_prefix(const FmhaParams& p, int* pre, int* wsum) {
    const int t = threadIdx.x, lane = t & 31, wid = t >> 5;
    int x = 0;
    if (t < p.batch) x = ragged_entry_tiles(ragged_clamp(__ldg(p.P_dev + t), p.rg_capacity), p.S, p.rg_units_per_entry);
    if (t < kRaggedMaxBatch) {
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) wsum[wid] = x;
    }
    __syncthreads();
    if (t < kRaggedMaxBatch) {
        int add = 0;
        for (int i = 0; i < wid; ++i) add += wsum[i];
        pre[t + 1] = x + add;
        if (t == 0) pre[0] = 0;
    }
}

// Copies the S block rows of kv head kv_z (K and V) into cache rows P..P+S-1, 16 bytes per
// thread-step, with `n` threads numbered `tid`.
__device__ __forceinline__ void append_block_rows(const FmhaParams& p, int D, int kv_z, int tid, int n) {
    const int vec_row = D / 8;
    const int per = p.S * vec_row;
    const size_t src0 = static_cast<size_t>(kv_z) * per;
    const size_t dst0 = (static_cast<size_t>(kv_z) * p.app_capacity + p.P) * vec_row;
    for (int i = tid; i < 2 * per; i += n) {
        const bool is_v = i >= per;
        const int e = is_v ? i - per : i;
        const uint4 x = __ldg((is_v ? p.app_src_v : p.app_src_k) + src0 + e);
        (is_v ? p.app_dst_v : p.app_dst_k)[dst0 + e] = x;
    }
}

template <int D, int MODE>
struct Cfg {
    static constexpr bool SAMPLE = (MODE == kDecoderSample);
    static constexpr int NQ = SAMPLE ? 1 : 2;                 // query tiles per work item
    static constexpr int NSB = SAMPLE ? 2 : 1;                // S buffers per query tile
    // Train calls at d <= 64 rotate three S buffers over both query tiles: S number n (counted
    // over the item sequence, both tiles interleaved) lives in buffer n % 3, so a query tile's
    // next S is computed while its softmax still works on the current one.  At d = 128 the two
    // O accumulators leave room for two S buffers only (one per query tile, NSB = 1).
    static constexpr bool ROT = !SAMPLE && D <= 64;
    static constexpr int NSBUF = ROT ? 3 : NQ * NSB;          // S buffers in TMEM, 128 columns each
    // s_full barriers: per S buffer, and with rotating buffers per (query tile, buffer), so that a
    // barrier's phases are one softmax warpgroup's S in that buffer, which it consumes in order.
    static constexpr int NSFULL = ROT ? NQ * 3 : NQ * NSB;
    static constexpr int O_COL = ROT ? 384 : 256;             // first TMEM column of the O sets
    static constexpr int NOB = ROT ? (D <= 32 ? 2 : 1) : (D <= 64 ? 2 : 1);  // O sets per query tile
    static_assert(O_COL + NOB * NQ * D <= 512, "TMEM columns");
    static constexpr int QBUF = (D == 128) ? 1 : 2;           // Q buffer sets (double-buffered)
    static constexpr int NST = SAMPLE ? (D == 128 ? 3 : (D == 64 ? 6 : 8)) : (D == 128 ? 2 : (D == 64 ? 4 : 6));
    static constexpr int RB = (D * 2 < 128) ? D * 2 : 128;  // bytes per smem row of one chunk
    static constexpr int NCH = D * 2 / RB;                   // column chunks per tile
    static constexpr uint32_t SWZ = (RB == 128) ? 2u : 4u;   // 128-byte / 64-byte swizzle
    static constexpr int CHUNK_BYTES = kBlockM * RB;
    static constexpr int TILE_BYTES = kBlockM * D * 2;
    static constexpr int KSTEPS_PER_CHUNK = RB / 32;         // 16-element k steps per chunk
    // Train calls stage the output tiles for a TMA store, except at d = 128 where the shared
    // memory is taken by the K/V ring; there rows are stored directly.
    static constexpr bool STAGE_O = !SAMPLE && (D <= 64);
};

template <int D, int MODE>
struct Smem {
    using C = Cfg<D, MODE>;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + C::QBUF * C::NQ * C::TILE_BYTES;
    static constexpr int OFF_V = OFF_K + C::NST * C::TILE_BYTES;
    static constexpr int OFF_O = OFF_V + C::NST * C::TILE_BYTES;
    static constexpr int O_BYTES = C::STAGE_O ? C::NQ * C::TILE_BYTES : 0;
    static constexpr int OFF_BAR = OFF_O + O_BYTES;
    // barriers: k_full[NST], v_full[NST], kv_empty[NST], q_full[QBUF], q_empty[QBUF],
    // s_full[NSFULL], p_full[NSBUF], pv_done[NQ][kPvRing], o_free[NOB*NQ], mma_drain, softmax_done
    static constexpr int NBAR = 3 * C::NST + 2 * C::QBUF + C::NSFULL + C::NSBUF + C::NQ * kPvRing + C::NOB * C::NQ + 2;
    static constexpr int OFF_MISC = ((OFF_BAR + NBAR * 8 + 15) / 16) * 16;
    // sampling: ragged prefix table pre[kRaggedMaxBatch + 1] and the scan's 8 warp sums
    static constexpr int OFF_RG = OFF_MISC + 64;
    static constexpr int RG_BYTES = C::SAMPLE ? ((kRaggedMaxBatch + 1 + 8) * 4 + 15) / 16 * 16 : 0;
    static constexpr int BYTES = OFF_RG + RG_BYTES;
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

// Sampling schedule.  The units (b, kv head, query tile) are taken in two phases: first the
// split units [0, split_units), whose key tiles form one stream cut into equal contiguous ranges
// for CTAs [0, split_ctas) (a unit whose tiles fall to several CTAs is merged by the last of them),
// then the whole units, unit split_units + k going to CTA k mod grid.  Whole units last means a
// CTA's final epilogue never waits for another CTA.
// A unit of work: NQ consecutive 128-row query tiles against a contiguous range of key tiles.
struct Item {
    int q_z;        // train: b*Hq + h (Q/O tensor-map z); sample: unit index
    int kv_z;       // b*Hkv + g
    int q_row0;     // train: first row (within the head) of query tile 0; sample: first packed row
    int q_y;        // TMA y coordinate of query tile 0
    int out_row0;   // sample: first row of the tile in the [B*Hq*S] row space
    int nact;       // query tiles with at least one valid row (1..NQ)
    int n1, a1;     // source-1 tiles (visited first), starting at key tile a1
    int n0;         // source-0 tiles, starting at key tile 0
    int t_begin, t_end;
    // sample: the unit's prefix length, its key tiles, its first tile in the stream of split
    // units, and the length of that stream
    int P, tu;
    long long ubeg, total;
    int sgrid;      // sample: CTAs the split stream is cut over
    // What each query tile needs of that stream: source-1 key tiles [a1q, e1q), source-0 key
    // tiles [0, n0q).  Other tiles are skipped for that query tile (no MMA, no softmax).
    int a1q[2], e1q[2], n0q[2];
};

// Key tile t of the item's stream is needed by query tile q.
__device__ __forceinline__ bool tile_needed(const Item& it, int q, int t) {
    // select, not index: q may be a runtime value and the arrays must stay in registers
    const int a1q = q ? it.a1q[1] : it.a1q[0];
    const int e1q = q ? it.e1q[1] : it.e1q[0];
    const int n0q = q ? it.n0q[1] : it.n0q[0];
    if (t < it.n1) {
        const int kt = it.a1 + t;
        return kt >= a1q && kt < e1q;
    }
    return (t - it.n1) < n0q;
}

// Key-tile ranges a block of query rows [r0, r_last] needs (train calls).
template <int MODE>
__device__ __forceinline__ void train_ranges(int L, int S, int r0, int r_last, int& a1, int& e1, int& n0) {
    if (MODE == kEncoder) {
        a1 = 0;
        e1 = 0;
        n0 = ceil_div_i(min(L, (r_last / S + 1) * S), kBlockN);
    } else {
        a1 = ((r0 / S) * S) / kBlockN;
        e1 = ceil_div_i(min(L, (r_last / S + 1) * S), kBlockN);
        n0 = ceil_div_i((r_last / S) * S, kBlockN);
    }
}

// Iterates the work items of this CTA.  Every role walks the same sequence.
//
// A ragged sampling call (P_dev set) has no whole-unit phase: the key tiles of every unit, entry
// b's units taking tiles pre[b]..pre[b+1]-1, form one stream cut into equal contiguous ranges for
// all gridDim.x CTAs; a CTA locates the unit of a tile by binary search over pre.
template <int MODE>
struct Scheduler {
    const FmhaParams& p;
    const int* rg_pre;   // sample, ragged: prefix table in shared memory
    long long pos, end;  // sample: tile range of this CTA
    long long total;     // sample: tiles of the split stream
    int sgrid;           // sample: CTAs the split stream is cut over
    int k;               // train: next item index (or next position in the item order)
    int k_end;           // train, item order: end of this CTA's positions
    const ItemOrder* ord;

    __device__ Scheduler(const FmhaParams& prm, const int* pre = nullptr, const ItemOrder* order = nullptr)
        : p(prm), rg_pre(pre), ord(order) {
        k = blockIdx.x;
        k_end = 0;
        if (MODE != kDecoderSample && ord != nullptr && ord->enabled) {
            k = ord->first[blockIdx.x];
            k_end = ord->first[blockIdx.x + 1];
        }
        if (MODE == kDecoderSample) {
            const int c = static_cast<int>(blockIdx.x);
            if (p.P_dev != nullptr) {
                // CTAs of the stream: one per unit at least, more while every CTA keeps about
                // kMinRaggedTiles tiles (a partial costs more than streaming a few tiles), never
                // more than the grid or the tile count (every CTA of the stream gets a tile)
                total = rg_pre[p.batch];
                const long long units = static_cast<long long>(p.batch) * p.rg_units_per_entry;
                long long g = total / kMinRaggedTiles;
                if (g < units) g = units;
                if (g > gridDim.x) g = gridDim.x;
                if (g > total) g = total;
                sgrid = static_cast<int>(g);
                pos = c < sgrid ? range_begin(c, total, sgrid) : 0;
                end = c < sgrid ? range_begin(c + 1, total, sgrid) : 0;
            } else {
                total = p.total_tiles;
                sgrid = p.split_ctas;
                pos = c < p.split_ctas ? range_begin(c, p.total_tiles, p.split_ctas) : 0;
                end = c < p.split_ctas ? range_begin(c + 1, p.total_tiles, p.split_ctas) : 0;
            }
        }
    }

    // Fills the sampling fields of unit u (prefix length P, Tu tiles, first stream tile ubeg).
    __device__ void fill_sample(Item& it, int u, int P, int Tu, long long ubeg, long long seg_begin,
                                long long seg_end) const {
        const int qt = u % p.num_qtiles;
        const int kvz = u / p.num_qtiles;  // b*Hkv + g
        const int b = kvz / p.kv_heads, g = kvz % p.kv_heads;
        it.q_z = u;
        it.kv_z = kvz;
        it.q_row0 = qt * kBlockM;
        it.out_row0 = (b * p.q_heads + g * p.group) * p.S + qt * kBlockM;
        it.q_y = it.out_row0;
        it.nact = 1;
        it.n1 = ceil_div_i(p.S, kBlockN);
        it.a1 = 0;
        it.n0 = ceil_div_i(P, kBlockN);
        it.a1q[0] = it.a1q[1] = 0;
        it.e1q[0] = it.e1q[1] = it.n1;
        it.n0q[0] = it.n0q[1] = it.n0;
        it.t_begin = static_cast<int>(seg_begin - ubeg);
        it.t_end = static_cast<int>(seg_end - ubeg);
        it.P = P;
        it.tu = Tu;
        it.ubeg = ubeg;
        it.total = total;
        it.sgrid = sgrid;
    }

    __device__ bool next(Item& it) {
        if (MODE == kDecoderSample && p.P_dev != nullptr) {
            if (pos >= end) return false;
            int lo = 0, hi = p.batch;  // pre[lo] <= pos < pre[hi]
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (rg_pre[mid] <= pos) lo = mid;
                else hi = mid;
            }
            const int UB = p.rg_units_per_entry;
            const int Tu = (rg_pre[lo + 1] - rg_pre[lo]) / UB;
            const int u_in = static_cast<int>((pos - rg_pre[lo]) / Tu);
            const long long ubeg = rg_pre[lo] + static_cast<long long>(u_in) * Tu;
            const long long seg_end = (end < ubeg + Tu) ? end : ubeg + Tu;
            fill_sample(it, lo * UB + u_in, ragged_clamp(__ldg(p.P_dev + lo), p.rg_capacity), Tu, ubeg, pos, seg_end);
            pos = seg_end;
            return true;
        }
        if (MODE == kDecoderSample) {
            const int Tu = p.tiles_per_unit;
            int u;
            long long ubeg, seg_end;
            if (pos < end) {
                u = static_cast<int>(pos / Tu);
                ubeg = static_cast<long long>(u) * Tu;
                seg_end = (end < ubeg + Tu) ? end : ubeg + Tu;
            } else if (k < p.whole_units) {
                u = p.split_units + k;
                k += gridDim.x;
                ubeg = 0;
                pos = 0;
                seg_end = Tu;
                end = 0;
            } else {
                return false;
            }
            fill_sample(it, u, p.P, Tu, ubeg, pos, seg_end);
            if (pos < end) pos = seg_end;
            return true;
        } else {
            int kk;
            if (ord != nullptr && ord->enabled) {
                if (k >= k_end) return false;
                kk = ord->item[k++];
            } else {
                if (k >= p.num_items) return false;
                kk = k;
                k += gridDim.x;
            }
            const int BH = p.batch * p.q_heads;
            const int qp = p.num_qtiles - 1 - kk / BH;  // pairs of query tiles, longest rows first
            const int bh = kk % BH;
            const int b = bh / p.q_heads, h = bh % p.q_heads;
            const int L = p.L, S = p.S;
            it.q_z = bh;
            it.kv_z = b * p.kv_heads + h / p.group;
            it.q_row0 = qp * 2 * kBlockM;
            it.q_y = it.q_row0;
            it.out_row0 = 0;
            it.nact = (it.q_row0 + kBlockM < L) ? 2 : 1;
            // Key tiles: each active query tile's ranges, and their union (the stream).
            int a1 = 1 << 30, e1 = 0, n0 = 0;
            for (int q = 0; q < 2; ++q) {
                const int r0 = it.q_row0 + q * kBlockM;
                if (q < it.nact) {
                    train_ranges<MODE>(L, S, r0, min(L, r0 + kBlockM) - 1, it.a1q[q], it.e1q[q], it.n0q[q]);
                    if (it.e1q[q] > it.a1q[q]) {
                        a1 = min(a1, it.a1q[q]);
                        e1 = max(e1, it.e1q[q]);
                    }
                    n0 = max(n0, it.n0q[q]);
                } else {
                    it.a1q[q] = it.e1q[q] = it.n0q[q] = 0;
                }
            }
            if (e1 == 0) a1 = 0;
            it.a1 = a1;
            it.n1 = e1 - a1;
            it.n0 = n0;
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
        const int len = (MODE == kDecoderSample) ? it.P : p.L;
        r.nk16 = round16(min(kBlockN, len - r.kt * kBlockN));
        r.box_rows = kBlockN;
    }
    return r;
}

// Limit of the pipeline waits (device variable, so that a test can shorten it without a rebuild;
// see e2d2_debug_set_wait_test) and a delay the producers of the next launches take before their
// first load (0 outside that test).
__device__ unsigned long long g_wait_limit_ns = kWaitTimeoutNs;
__device__ unsigned long long g_test_producer_delay_ns = 0;

// Bounded mbarrier wait.  Returns false (and flags the CTA and the device error word) if the
// phase does not complete within the limit or another role already gave up.  The thread sleeps
// inside try_wait (up to 1 ms per attempt) rather than spinning.  Pipeline waits use the
// (test-adjustable) limit g_wait_limit_ns; drain waits (`drain`: the last copies of a producer,
// the MMAs and roles that must be done before tensor memory is freed) always allow kWaitTimeoutNs,
// so a shortened limit never frees resources that are still in use.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         unsigned int* err, bool drain = false) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    unsigned long long limit = kWaitTimeoutNs + 0ull;
    if (!drain) limit = *reinterpret_cast<volatile unsigned long long*>(&g_wait_limit_ns);
    const uint64_t t0 = ptx::globaltimer_ns();
    for (;;) {
        if (ptx::mbar_try_wait_sleep(bar, parity, 1000000u)) return true;
        if (*abort_flag) return false;
        if (ptx::globaltimer_ns() - t0 > limit) {
            *abort_flag = 1;
            atomicOr(err, kErrWaitTimeout);
            return false;
        }
    }
}

// Warp-collective form of wait_bar: every lane returns the same answer, so the .sync.aligned
// tcgen05 instructions that follow are always executed by the whole warp.
__device__ __forceinline__ bool wait_bar_warp(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              unsigned int* err, bool drain = false) {
    const bool ok = wait_bar(bar, parity, abort_flag, err, drain);
    return __all_sync(0xffffffffu, ok);
}

// Test hook: the producer sleeps for g_test_producer_delay_ns before its first load (bounded).
__device__ __forceinline__ void test_producer_delay() {
    const unsigned long long delay = *reinterpret_cast<volatile unsigned long long*>(&g_test_producer_delay_ns);
    if (delay == 0) return;
    const uint64_t t0 = ptx::globaltimer_ns();
    while (ptx::globaltimer_ns() - t0 < delay) __nanosleep(100000);
}

// Byte offset of 16-byte unit `u` of row `r` inside one swizzled chunk (row pitch RB bytes).
template <int RB>
__device__ __forceinline__ uint32_t swz_offset(int r, int u) {
    const uint32_t a = static_cast<uint32_t>(r * RB + u * 16);
    constexpr uint32_t mask = (RB == 128) ? 7u : 3u;
    return a ^ (((a >> 7) & mask) << 4);
}

// TMEM column (relative to the S buffer) holding the packed bf16 P of keys 16ks..16ks+15 (two
// keys per 32-bit column, over S columns 0-63; the softmax reads all of S before writing P).
__device__ __forceinline__ uint32_t p_col(uint32_t ks) { return ks * 8; }

// A P.V that waits for its softmax: the key tile it belongs to and where its operands live.
struct PendingPV {
    bool have;
    bool first;        // first tile of its item: overwrite O, wait for the O buffer to be free
    int q;             // query tile
    uint32_t st;       // K/V stage
    uint32_t round;    // stage round (v_full parity)
    uint32_t qt;       // S buffer use: per-query-tile tile counter, or (rotating buffers) S number
    uint32_t qi;       // per-query-tile item counter (o_free parity, O buffer)
    uint32_t nk;       // keys in the tile (multiple of 16)
    uint32_t pvn;      // P.V number of its query tile (pv_done ring slot pvn % kPvRing)
};

// Issues O[q] (+)= P[q] . V[st] (A = P from TMEM, B = V MN-major in shared memory) once the
// softmax of query tile q has published P, the O buffer is free (first tile of an item) and V
// has landed; then releases the K/V stage (kv_empty) for this query tile.
template <class C>
__device__ __forceinline__ bool issue_pv(int q, const PendingPV& pv, uint64_t* p_full, uint64_t* o_free,
                                         uint64_t* v_full, uint64_t* kv_empty, uint64_t* pv_done,
                                         volatile int* abort_flag, unsigned int* err, uint32_t tmem_base,
                                         uint32_t sV, uint64_t vdesc, uint32_t idesc_pv, int D, bool leader) {
    const uint32_t sb = C::ROT ? pv.qt % 3 : q * C::NSB + pv.qt % C::NSB;
    const uint32_t sph = C::ROT ? (pv.qt / 3) & 1 : (pv.qt / C::NSB) & 1;
    if (!wait_bar_warp(&p_full[sb], sph, abort_flag, err)) return false;
    const uint32_t ob = pv.qi % C::NOB;
    if (pv.first && !wait_bar_warp(&o_free[ob * C::NQ + q], ((pv.qi / C::NOB) & 1) ^ 1, abort_flag, err))
        return false;
    if (!wait_bar_warp(&v_full[pv.st], pv.round & 1, abort_flag, err)) return false;
    ptx::tc_fence_after();
    if (leader) {
        const uint32_t a_tmem = tmem_base + sb * 128;
        const uint32_t d_tmem = tmem_base + C::O_COL + (ob * C::NQ + q) * D;
        const uint32_t v_base = sV + pv.st * C::TILE_BYTES;
        for (uint32_t ks = 0; ks < pv.nk / 16; ++ks)
            ptx::mma_ts(d_tmem, a_tmem + p_col(ks), vdesc | ((v_base + ks * 16 * C::RB) >> 4), idesc_pv,
                        (pv.first && ks == 0) ? 0u : 1u);
        ptx::mma_commit(&pv_done[q * kPvRing + pv.pvn % kPvRing]);
        ptx::mma_commit(&kv_empty[pv.st]);
    }
    __syncwarp();
    return true;
}

// Loads N consecutive fp32 TMEM columns of this thread's lane (N in {16, 32}).
template <int N>
__device__ __forceinline__ void load_tmem_cols(uint32_t taddr, float* o) {
    uint32_t r[N];
    if constexpr (N == 16) {
        ptx::tmem_ld16(taddr, *reinterpret_cast<uint32_t(*)[16]>(r));
    } else {
        ptx::tmem_ld32(taddr, r);
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

// Loads the 128 S columns of this thread's row (one TMEM round trip, eight 16-column loads),
// applies the row's key interval [cmin, cmax) (tile-relative) and sets chunks without any allowed
// key in the warp (live bit clear) to -inf.  The loads are unconditional so that s has a single
// definition (no spills).  Returns the row maximum.
__device__ __forceinline__ float load_s_row(uint32_t s_tmem, uint32_t live, int cmin, int cmax, float (&s)[128]) {
    uint32_t raw[128];
#pragma unroll
    for (int h = 0; h < 8; ++h) ptx::tmem_ld16(s_tmem + 16 * h, *reinterpret_cast<uint32_t(*)[16]>(&raw[16 * h]));
    ptx::tmem_wait_ld();
    ptx::reg_fence<128>(raw);
#pragma unroll
    for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(raw[c]);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        if (!(live & (1u << a))) {
#pragma unroll
            for (int c = 0; c < 32; ++c) s[32 * a + c] = -INFINITY;
        } else if (!__all_sync(0xffffffffu, cmin <= 32 * a && cmax >= 32 * a + 32)) {
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const int col = 32 * a + c;
                s[col] = (col >= cmin && col < cmax) ? s[col] : -INFINITY;
            }
        }
    }
    // maximum as a tree: eight independent chains over 16 columns each, then 8 -> 3 -> 1
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = s[j];
#pragma unroll
    for (int c = 8; c < 120; c += 16)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = ptx::fmax3(acc[j], s[c + j], s[c + 8 + j]);
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = fmaxf(acc[j], s[120 + j]);
    return ptx::fmax3(ptx::fmax3(acc[0], acc[1], acc[2]), ptx::fmax3(acc[3], acc[4], acc[5]), fmaxf(acc[6], acc[7]));
}

// P = exp2(s * sl2 + neg_m) for the live chunks, packed to bf16 and stored over S (keys 32a..
// 32a+31 -> columns 16a..16a+15); dead chunks below nchunks store zeros.  Returns the row sum.
// The arguments and the sums run on column pairs (packed fp32x2 FMA / add of sm_100), the
// exponentials one by one.
__device__ __forceinline__ float exp_store_row(uint32_t s_tmem, uint32_t live, int nchunks, const float (&s)[128],
                                               float sl2, float neg_m) {
    const float2 sl2v = make_float2(sl2, sl2), nm = make_float2(neg_m, neg_m);
    float2 sums[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        if (a < nchunks) {
            uint32_t pk[16];
            if (live & (1u << a)) {
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const float2 x = __ffma2_rn(make_float2(s[32 * a + c], s[32 * a + c + 1]), sl2v, nm);
                    const float2 e = make_float2(ptx::ex2(x.x), ptx::ex2(x.y));
                    sums[(c >> 1) & 1] = __fadd2_rn(sums[(c >> 1) & 1], e);
                    pk[c / 2] = ptx::pack_bf16x2(e.x, e.y);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 16; ++c) pk[c] = 0u;
            }
            ptx::tmem_st16(s_tmem + p_col(2 * a), pk);
        }
    }
    const float2 t = __fadd2_rn(sums[0], sums[1]);
    return t.x + t.y;
}

template <int MODE>
__device__ __forceinline__ const ItemOrder* order_ptr(const ItemOrder& o) {
    return &o;
}
template <int MODE>
__device__ __forceinline__ const ItemOrder* order_ptr(const NoOrder&) {
    return nullptr;
}

template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, 1) fmha_sm100_kernel(const __grid_constant__ FmhaParams p,
                                                                  const __grid_constant__ typename OrderOf<MODE>::type ord) {
    using C = Cfg<D, MODE>;
    using SM = Smem<D, MODE>;
    constexpr int NQ = C::NQ, NSB = C::NSB, NOB = C::NOB;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    ptx::griddep_launch_dependents();  // the next kernel may launch; it waits for this one's end
    // All shared-memory pointers derive from `smem`; the roles recompute them after setmaxnreg
    // so that nothing but smem/tmem_base lives across the register-budget change.
#define E2D2_SMEM_POINTERS                                                                           \
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &      \
                                               ~static_cast<uintptr_t>(1023));                       \
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::OFF_BAR);                                \
    uint64_t* k_full = bars;                                                                         \
    uint64_t* v_full = bars + C::NST;                                                                \
    uint64_t* kv_empty = bars + 2 * C::NST;                                                          \
    uint64_t* q_full = bars + 3 * C::NST;                                                            \
    uint64_t* q_empty = q_full + C::QBUF;                                                            \
    uint64_t* s_full = q_empty + C::QBUF;  /* [S buffer] or [q][S buffer] */                         \
    uint64_t* p_full = s_full + C::NSFULL; /* [S buffer] */                                          \
    uint64_t* pv_done = p_full + C::NSBUF; /* [q][kPvRing] */                                        \
    uint64_t* o_free = pv_done + NQ * kPvRing; /* [ob][q] */                                         \
    uint64_t* mma_drain = o_free + NOB * NQ;                                                         \
    uint64_t* softmax_done = mma_drain + 1; /* every softmax thread is finished with TMEM */        \
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SM::OFF_MISC);                        \
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM::OFF_MISC + 8);             \
    volatile int* bcast = reinterpret_cast<volatile int*>(smem + SM::OFF_MISC + 16);                 \
    int* rg_pre = reinterpret_cast<int*>(smem + SM::OFF_RG);                                         \
    (void)rg_pre;                                                                                    \
    (void)k_full; (void)v_full; (void)kv_empty; (void)q_full; (void)q_empty; (void)s_full;           \
    (void)p_full; (void)pv_done; (void)o_free; (void)mma_drain; (void)tmem_holder; (void)abort_flag; \
    (void)softmax_done;                                                                              \
    (void)bcast;
    uint32_t tmem_base;
    {
    E2D2_SMEM_POINTERS
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NST; ++i) {
            ptx::mbar_init(&k_full[i], 1);
            ptx::mbar_init(&v_full[i], 1);
            ptx::mbar_init(&kv_empty[i], NQ);
        }
        for (int i = 0; i < C::QBUF; ++i) {
            ptx::mbar_init(&q_full[i], 1);
            ptx::mbar_init(&q_empty[i], 1);
        }
        for (int i = 0; i < C::NSFULL; ++i) ptx::mbar_init(&s_full[i], 1);
        for (int i = 0; i < C::NSBUF; ++i) ptx::mbar_init(&p_full[i], kSoftmaxThreads / 2);
        for (int i = 0; i < NQ * kPvRing; ++i) ptx::mbar_init(&pv_done[i], 1);
        for (int i = 0; i < NOB * NQ; ++i) ptx::mbar_init(&o_free[i], kSoftmaxThreads / 2);
        ptx::mbar_init(mma_drain, 1);
        ptx::mbar_init(softmax_done, kSoftmaxThreads);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_holder, kTmemCols);
        ptx::tmem_relinquish();
    }
    // Everything above touches only this CTA's resources; inputs are read after the previous
    // kernel on the stream has finished (programmatic dependent launch).
    ptx::griddep_wait();
    if (MODE == kDecoderSample && p.P_dev != nullptr) ragged_prefix(p, rg_pre, rg_pre + kRaggedMaxBatch + 1);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    tmem_base = *tmem_holder;
    }

    E2D2_SMEM_POINTERS
    const uint32_t smem_base = ptx::smem_u32(smem);
    const uint32_t sQ = smem_base + SM::OFF_Q;
    const uint32_t sK = smem_base + SM::OFF_K;
    const uint32_t sV = smem_base + SM::OFF_V;

    if (warp == 0) {
        ptx::setmaxnreg_dec<kRegsControl>();
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
        test_producer_delay();
        Scheduler<MODE> sched(p, rg_pre, order_ptr<MODE>(ord));
        Item it;
        uint32_t kv_iter = 0, item_idx = 0;
        bool ok = true;
        while (ok && sched.next(it)) {
            const int qb = item_idx % C::QBUF;
            const uint32_t qround = item_idx / C::QBUF;
            ok = wait_bar_warp(&q_empty[qb], (qround & 1) ^ 1, abort_flag, p.err);
            if (!ok) break;
            E2D2_DCHECK(MODE == kDecoderSample ? (it.q_z < p.batch * p.kv_heads * p.num_qtiles && it.q_row0 < p.rows_per_unit)
                                               : (it.q_z < p.batch * p.q_heads && it.q_y < p.L),
                        p.err);
            if (leader) {
                if (MODE == kDecoderSample) {
                    // The packed rows are spread over the four TMEM lane quarters: rows
                    // [k*q_chunk, (k+1)*q_chunk) go to tile rows 32k.. so that every softmax warp
                    // gets a share of them.
                    ptx::mbar_arrive_expect_tx(&q_full[qb], 4u * p.q_chunk * D * 2);
                    for (int k = 0; k < 4; ++k)
                        for (int ch = 0; ch < C::NCH; ++ch) {
                            uint8_t* dst = smem + SM::OFF_Q + qb * C::TILE_BYTES + ch * C::CHUNK_BYTES + 32 * k * C::RB;
                            ptx::tma_load_2d(&p.tm_q, &q_full[qb], dst, ch * (C::RB / 2), it.q_y + k * p.q_chunk);
                        }
                } else {
                    ptx::mbar_arrive_expect_tx(&q_full[qb], NQ * C::TILE_BYTES);
                    for (int q = 0; q < NQ; ++q)
                        for (int ch = 0; ch < C::NCH; ++ch) {
                            uint8_t* dst = smem + SM::OFF_Q + (qb * NQ + q) * C::TILE_BYTES + ch * C::CHUNK_BYTES;
                            ptx::tma_load_3d(&p.tm_q, &q_full[qb], dst, ch * (C::RB / 2), it.q_y + q * kBlockM,
                                             it.q_z);
                        }
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
                // debug builds: the tile starts inside its source and the kv unit exists
                E2D2_DCHECK(tr.kt * kBlockN < (tr.src ? (MODE == kDecoderSample ? p.S : p.L)
                                                      : (MODE == kDecoderSample ? it.P : p.L)),
                            p.err);
                E2D2_DCHECK(it.kv_z >= 0 && it.kv_z < p.batch * p.kv_heads, p.err);
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
        // NST K/V loads and the last QBUF Q loads).
        volatile int no_abort = 0;
        const uint32_t first_live = kv_iter > static_cast<uint32_t>(C::NST) ? kv_iter - C::NST : 0u;
        for (uint32_t i = first_live; i < kv_iter; ++i) {
            wait_bar_warp(&k_full[i % C::NST], (i / C::NST) & 1u, &no_abort, p.err, true);
            wait_bar_warp(&v_full[i % C::NST], (i / C::NST) & 1u, &no_abort, p.err, true);
        }
        for (uint32_t i = item_idx > static_cast<uint32_t>(C::QBUF) ? item_idx - C::QBUF : 0u; i < item_idx; ++i)
            wait_bar_warp(&q_full[i % C::QBUF], (i / C::QBUF) & 1u, &no_abort, p.err, true);
    } else if (warp == 1) {
        ptx::setmaxnreg_dec<kRegsControl>();
        // ------------------------------------------------------------------ MMA issuer
        // The whole warp walks the schedule, so descriptors and TMEM addresses are warp-uniform;
        // one elected lane issues tcgen05.mma / tcgen05.commit.
        const bool leader = ptx::elect_one();
        Scheduler<MODE> sched(p, rg_pre, order_ptr<MODE>(ord));
        Item it;
        uint32_t kv_iter = 0, item_idx = 0;
        uint32_t qtile[NQ], qitem[NQ];
        PendingPV pend[NQ];
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
            qtile[q] = qitem[q] = 0;
            pend[q].have = false;
        }
        // Descriptor bits without the start address (added per MMA).
        const uint64_t kdesc = ptx::smem_desc(0, 16, 8 * C::RB, C::SWZ);             // Q, K: K-major
        const uint64_t vdesc = ptx::smem_desc(0, C::CHUNK_BYTES, 8 * C::RB, C::SWZ);  // V: MN-major
        constexpr uint32_t idesc_pv = ptx::idesc_bf16_f32(kBlockM, D, true);
        bool ok = true;
        if constexpr (C::ROT) {
            // Rotating S buffers.  S number n goes to buffer n % 3, whose previous S (n - 3) is
            // consumed by its P.V: that P.V is issued first (the tensor core runs one CTA's MMAs
            // in order, so the P.V reads P before the new S overwrites it).  The P.V still owed
            // are kept in issue order, at most three (f0 oldest).
            PendingPV f0, f1, f2;
            f0.have = f1.have = f2.have = false;
            int nf = 0;
            uint32_t seq = 0;
            uint32_t qitem[NQ], qpv[NQ];
#pragma unroll
            for (int q = 0; q < NQ; ++q) qitem[q] = qpv[q] = 0;
            auto pop = [&]() -> bool {
                const bool r = issue_pv<C>(f0.q, f0, p_full, o_free, v_full, kv_empty, pv_done, abort_flag, p.err,
                                           tmem_base, sV, vdesc, idesc_pv, D, leader);
                f0 = f1;
                f1 = f2;
                --nf;
                return r;
            };
            while (ok && sched.next(it)) {
                const int qb = item_idx % C::QBUF;
                ok = wait_bar_warp(&q_full[qb], (item_idx / C::QBUF) & 1, abort_flag, p.err);
                if (!ok) break;
                bool seen[NQ];
#pragma unroll
                for (int q = 0; q < NQ; ++q) seen[q] = false;
                for (int t = it.t_begin; t < it.t_end && ok; ++t) {
                    const uint32_t st = kv_iter % C::NST;
                    const uint32_t round = kv_iter / C::NST;
                    // The stage is reloaded only after the P.V that still reads its old V.
                    while (ok && ((nf > 0 && f0.st == st) || (nf > 1 && f1.st == st) || (nf > 2 && f2.st == st)))
                        ok = pop();
                    if (!ok) break;
                    ok = wait_bar_warp(&k_full[st], round & 1, abort_flag, p.err);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    const TileRef tr = tile_of<MODE>(p, it, t);
                    const uint32_t idesc_qk = ptx::idesc_bf16_f32(kBlockM, tr.nk16, false);
                    const uint32_t k_base = sK + st * C::TILE_BYTES;
#pragma unroll
                    for (int q = 0; q < NQ; ++q) {
                        if (q >= it.nact || !tile_needed(it, q, t)) {
                            if (leader) ptx::mbar_arrive(&kv_empty[st]);
                            __syncwarp();
                            continue;
                        }
                        while (ok && nf > 0 && f0.qt + 3 <= seq) ok = pop();
                        if (!ok) break;
                        const uint32_t sb = seq % 3;
                        if (leader) {
                            const uint32_t q_base = sQ + (qb * NQ + q) * C::TILE_BYTES;
#pragma unroll
                            for (int ks = 0; ks < D / 16; ++ks) {
                                const uint32_t off = (ks / C::KSTEPS_PER_CHUNK) * C::CHUNK_BYTES +
                                                     (ks % C::KSTEPS_PER_CHUNK) * 32;
                                ptx::mma_ss(tmem_base + sb * 128, kdesc | ((q_base + off) >> 4),
                                            kdesc | ((k_base + off) >> 4), idesc_qk, ks > 0 ? 1u : 0u);
                            }
                            ptx::mma_commit(&s_full[q * 3 + sb]);
                        }
                        __syncwarp();
                        PendingPV e;
                        e.have = true;
                        e.first = !seen[q];
                        e.q = q;
                        e.st = st;
                        e.round = round;
                        e.qt = seq;
                        e.qi = qitem[q];
                        e.nk = tr.nk16;
                        e.pvn = qpv[q]++;
                        if (nf == 0) f0 = e;
                        else if (nf == 1) f1 = e;
                        else f2 = e;
                        ++nf;
                        ++seq;
                        seen[q] = true;
                    }
                    ++kv_iter;
                }
#pragma unroll
                for (int q = 0; q < NQ; ++q)
                    if (q < it.nact) ++qitem[q];
                if (leader) ptx::mma_commit(&q_empty[qb]);
                __syncwarp();
                ++item_idx;
                // The item's last P.V go out as soon as their P is ready: the epilogues wait for
                // them (left queued, they would wait for the next item's S).
                while (ok && nf > 0) ok = pop();
            }
        } else {
            while (ok && sched.next(it)) {
                const int qb = item_idx % C::QBUF;
                ok = wait_bar_warp(&q_full[qb], (item_idx / C::QBUF) & 1, abort_flag, p.err);
                if (!ok) break;
                // A query tile that sits this item out gets its last P.V issued now.
    #pragma unroll
                for (int q = 0; q < NQ; ++q)
                    if (q >= it.nact && pend[q].have) {
                        ok = ok && issue_pv<C>(q, pend[q], p_full, o_free, v_full, kv_empty, pv_done, abort_flag, p.err,
                                               tmem_base, sV, vdesc, idesc_pv, D, leader);
                        pend[q].have = false;
                    }
                if (!ok) break;
                bool seen[NQ];
    #pragma unroll
                for (int q = 0; q < NQ; ++q) seen[q] = false;
                for (int t = it.t_begin; t < it.t_end && ok; ++t) {
                    const uint32_t st = kv_iter % C::NST;
                    const uint32_t round = kv_iter / C::NST;
                    // A P.V still pending on this stage (its query tile skipped the tiles since)
                    // must be issued now: the stage is reloaded only after it.
    #pragma unroll
                    for (int q = 0; q < NQ; ++q)
                        if (ok && pend[q].have && pend[q].st == st) {
                            ok = issue_pv<C>(q, pend[q], p_full, o_free, v_full, kv_empty, pv_done, abort_flag, p.err,
                                             tmem_base, sV, vdesc, idesc_pv, D, leader);
                            pend[q].have = false;
                        }
                    if (!ok) break;
                    ok = wait_bar_warp(&k_full[st], round & 1, abort_flag, p.err);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    const TileRef tr = tile_of<MODE>(p, it, t);
                    const uint32_t idesc_qk = ptx::idesc_bf16_f32(kBlockM, tr.nk16, false);
                    const uint32_t k_base = sK + st * C::TILE_BYTES;
    #pragma unroll
                    for (int q = 0; q < NQ; ++q) {
                        if (q >= it.nact || !tile_needed(it, q, t)) {
                            // This query tile does not use the stage: its kv_empty share is free now.
                            if (leader) ptx::mbar_arrive(&kv_empty[st]);
                            __syncwarp();
                            continue;
                        }
                        const uint32_t sbuf = qtile[q] % NSB;
                        // With one S buffer per query tile, the pending P.V (reading P over S) must be
                        // issued before S is overwritten; with two, S first keeps the tensor core busy.
                        if (NSB == 1 && pend[q].have) {
                            ok = issue_pv<C>(q, pend[q], p_full, o_free, v_full, kv_empty, pv_done, abort_flag, p.err,
                                             tmem_base, sV, vdesc, idesc_pv, D, leader);
                            if (!ok) break;
                        }
                        if (leader) {
                            const uint32_t q_base = sQ + (qb * NQ + q) * C::TILE_BYTES;
    #pragma unroll
                            for (int ks = 0; ks < D / 16; ++ks) {
                                const uint32_t off = (ks / C::KSTEPS_PER_CHUNK) * C::CHUNK_BYTES +
                                                     (ks % C::KSTEPS_PER_CHUNK) * 32;
                                ptx::mma_ss(tmem_base + (q * NSB + sbuf) * 128, kdesc | ((q_base + off) >> 4),
                                            kdesc | ((k_base + off) >> 4), idesc_qk, ks > 0 ? 1u : 0u);
                            }
                            ptx::mma_commit(&s_full[q * NSB + sbuf]);
                        }
                        __syncwarp();
                        if (NSB == 2 && pend[q].have) {
                            ok = issue_pv<C>(q, pend[q], p_full, o_free, v_full, kv_empty, pv_done, abort_flag, p.err,
                                             tmem_base, sV, vdesc, idesc_pv, D, leader);
                            if (!ok) break;
                        }
                        pend[q].have = true;
                        pend[q].first = !seen[q];
                        seen[q] = true;
                        pend[q].st = st;
                        pend[q].round = round;
                        pend[q].qt = qtile[q];
                        pend[q].qi = qitem[q];
                        pend[q].nk = tr.nk16;
                        pend[q].pvn = qtile[q];
                        ++qtile[q];
                    }
                    ++kv_iter;
                }
    #pragma unroll
                for (int q = 0; q < NQ; ++q)
                    if (q < it.nact) ++qitem[q];
                // Q of this item is free once every QK^T issued so far has completed.
                if (leader) ptx::mma_commit(&q_empty[qb]);
                __syncwarp();
                ++item_idx;
            }
    #pragma unroll
            for (int q = 0; q < NQ; ++q)
                if (ok && pend[q].have)
                    ok = issue_pv<C>(q, pend[q], p_full, o_free, v_full, kv_empty, pv_done, abort_flag, p.err, tmem_base,
                                     sV, vdesc, idesc_pv, D, leader);
        }
        // Drain: every MMA issued by this warp completes, and every softmax thread is done with
        // TMEM, before TMEM is released.
        if (leader) ptx::mma_commit(mma_drain);
        __syncwarp();
        volatile int no_abort = 0;
        wait_bar_warp(mma_drain, 0, &no_abort, p.err, true);
        wait_bar_warp(softmax_done, 0, &no_abort, p.err, true);
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, kTmemCols);
    } else if (warp < 4) {
        ptx::setmaxnreg_dec<kRegsControl>();
        // Warps 2-3: the cache write of an encoder block step (sampling calls only), else idle.
        if (MODE == kDecoderSample && p.app_dst_k != nullptr) {
            Scheduler<MODE> sched(p, rg_pre, order_ptr<MODE>(ord));
            Item it;
            while (sched.next(it))
                if (it.t_begin == 0 && it.q_row0 == 0) append_block_rows(p, D, it.kv_z, threadIdx.x - 64, 64);
        }
    } else {
        ptx::setmaxnreg_inc<kRegsSoftmax>();
        // ------------------------------------------------------------------ softmax warpgroups
        // Warpgroup 1+q (warps 4+4q .. 7+4q) owns query tile q; each thread one row (its TMEM
        // lane) and all key columns.  Waits never break these loops: every warp takes every
        // named barrier, so a wait that gives up (device error word set) cannot strand another.
        const int q = (warp - 4) >> 2;
        const int quarter = warp & 3;                // TMEM lane quarter
        const int row = quarter * 32 + lane;         // row of the query tile
        const int wtid = threadIdx.x - 128 - 128 * q; // 0..127 within the warpgroup
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t wg_bar = 1 + q;               // named barrier of this warpgroup
        const float sl2 = p.scale_log2;
        if (q < NQ) {
            Scheduler<MODE> sched(p, rg_pre, order_ptr<MODE>(ord));
            Item it;
            uint32_t qtile = 0, qitem = 0;
            uint32_t seq = 0;     // rotating S buffers: S numbers issued so far (both query tiles)
            uint32_t s_par = 0;   // rotating S buffers: bit b = parity of this tile's next S in buffer b
            while (sched.next(it)) {
                if (q >= it.nact) {
                    // No valid row in this query tile: nothing to do but count the other's S.
                    if (C::ROT)
                        for (int t = it.t_begin; t < it.t_end; ++t) seq += tile_needed(it, 0, t) ? 1u : 0u;
                    continue;
                }
                // Per-row key intervals [lo, hi) for source 0 and source 1 (empty for padded rows).
                int lo0, hi0, lo1, hi1;
                bool row_valid;
                // Row of this lane within the head (train) or within the packed tile (sample: lane
                // quarter k holds packed rows k*q_chunk ..).
                const int prow = (MODE == kDecoderSample) ? (lane < p.q_chunk ? quarter * p.q_chunk + lane : kBlockM)
                                                          : row;
                const int qrow = it.q_row0 + q * kBlockM + prow;
                if (MODE == kDecoderSample) {
                    row_valid = prow < kBlockM && qrow < p.rows_per_unit;
                    lo0 = 0;
                    hi0 = row_valid ? it.P : 0;
                    lo1 = 0;
                    hi1 = row_valid ? p.S : 0;
                } else {
                    row_valid = qrow < p.L;
                    const int i = min(qrow, p.L - 1);
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
                float m = -INFINITY, l = 0.f;  // running max (log2 units) and sum of this row
                const uint32_t ob = qitem % NOB;
                const uint32_t o_tmem = tmem_base + lane_off + C::O_COL + (ob * NQ + q) * D;
                bool first = true;
                for (int t = it.t_begin; t < it.t_end; ++t) {
                    uint32_t my_seq = 0;
                    if (C::ROT) {
                        // the MMA warp numbers the S of a key tile query tile 0 first
                        const bool n0 = tile_needed(it, 0, t);
                        const bool n1 = it.nact > 1 && tile_needed(it, 1, t);
                        my_seq = seq + ((q == 1 && n0) ? 1u : 0u);
                        seq += (n0 ? 1u : 0u) + (n1 ? 1u : 0u);
                    }
                    if (!tile_needed(it, q, t)) continue;
                    const uint32_t sbuf = C::ROT ? my_seq % 3 : q * NSB + qtile % NSB;
                    const uint32_t sph = C::ROT ? (s_par >> sbuf) & 1u : (qtile / NSB) & 1;
                    if (C::ROT) s_par ^= 1u << sbuf;
                    wait_bar_warp(&s_full[C::ROT ? q * 3 + sbuf : sbuf], sph, abort_flag, p.err);
                    ptx::tc_fence_after();
                    const TileRef tr = tile_of<MODE>(p, it, t);
                    const int k0 = tr.kt * kBlockN;
                    const int lo = tr.src ? lo1 : lo0;
                    const int hi = tr.src ? hi1 : hi0;
                    const int cmin = lo - k0;
                    const int cmax = min(hi - k0, tr.nk16);
                    const int nchunks = (tr.nk16 + 31) / 32;
                    const uint32_t s_tmem = tmem_base + lane_off + sbuf * 128;
                    // live: some row of the warp has an allowed key in the 32-column chunk.
                    uint32_t live = 0;
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        const bool mine = (a < nchunks) && (cmin < 32 * a + 32) && (cmax > 32 * a);
                        if (__any_sync(0xffffffffu, mine)) live |= 1u << a;
                    }
                    float s[128];
                    const float mx = load_s_row(s_tmem, live, cmin, cmax, s);
                    const float m_new = fmaxf(m, mx * sl2);
                    bool rescale = false;
                    float alpha = 1.f;
                    if (m_new > m + kRescaleThreshold) {
                        alpha = ptx::ex2(m - m_new);
                        rescale = !first;
                        m = m_new;
                        l *= alpha;
                    }
                    const float neg_m = (m == -INFINITY) ? 0.f : -m;
                    l += exp_store_row(s_tmem, live, nchunks, s, sl2, neg_m);
                    // tcgen05.ld/st are warp-collective: the warp rescales if any row needs it, and O may
                    // only be touched once the previous P.V has landed (without a rescale there is
                    // nothing to wait for: see kPvRing).
                    if (!first && __any_sync(0xffffffffu, rescale)) {
                        wait_bar_warp(&pv_done[q * kPvRing + (qtile - 1) % kPvRing], ((qtile - 1) / kPvRing) & 1,
                                      abort_flag, p.err);
                        ptx::tc_fence_after();
                        rescale_tmem_cols<D>(o_tmem, rescale ? alpha : 1.f);
                    }
                    if (MODE == kDecoderSample && p.P_dev != nullptr && tr.src == 0 && it.P - k0 < tr.nk16) {
                        // Ragged prefix: cache rows at or past P[b] in this tile may hold anything (NaN
                        // included) and P.V would meet them with p = 0; zero those V rows of the stage.
                        const uint32_t vst = qtile % C::NST;
                        wait_bar_warp(&v_full[vst], (qtile / C::NST) & 1u, abort_flag, p.err);
                        const int vrow = quarter * 32 + lane;
                        if (vrow >= it.P - k0 && vrow < tr.nk16) {
#pragma unroll
                            for (int ch = 0; ch < C::NCH; ++ch) {
                                uint4* dst = reinterpret_cast<uint4*>(smem + SM::OFF_V + vst * C::TILE_BYTES +
                                                                      ch * C::CHUNK_BYTES + vrow * C::RB);
#pragma unroll
                                for (int u = 0; u < C::RB / 16; ++u) dst[u] = make_uint4(0u, 0u, 0u, 0u);
                            }
                        }
                        ptx::fence_proxy_async_smem();
                    }
                    ptx::tmem_wait_st();
                    ptx::tc_fence_before();
                    ptx::mbar_arrive(&p_full[sbuf]);
                    ++qtile;
                    first = false;
                }
                // ------------------------------------------------------------ epilogue
                wait_bar_warp(&pv_done[q * kPvRing + (qtile - 1) % kPvRing], ((qtile - 1) / kPvRing) & 1, abort_flag,
                              p.err);
                ptx::tc_fence_after();
                const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
                const float lse_val = (l > 0.f) ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
                constexpr int CW = D < 32 ? D : 32;  // columns per step
                __nv_bfloat16* outp = reinterpret_cast<__nv_bfloat16*>(p.out);
                const int Tu = it.tu;
                const bool whole = (MODE != kDecoderSample) || (it.t_begin == 0 && it.t_end == Tu);
                float* slot = nullptr;
                int c_first = 0, c_last = 0;
                long long ubeg = 0;
                if (MODE == kDecoderSample && !whole) {
                    ubeg = it.ubeg;
                    c_first = owner_cta(ubeg, it.total, it.sgrid);
                    c_last = owner_cta(ubeg + Tu - 1, it.total, it.sgrid);
                    const int my_slot = (range_begin(blockIdx.x, it.total, it.sgrid) >= ubeg)
                                            ? 2 * blockIdx.x
                                            : 2 * blockIdx.x + 1;
                    slot = p.ws_partial + static_cast<size_t>(my_slot) * p.slot_floats;
                }
                uint8_t* stage = smem + SM::OFF_O + q * C::TILE_BYTES;
                if (C::STAGE_O) {
                    if (wtid == 0) ptx::tma_store_wait_read_all();
                    ptx::named_barrier_sync(wg_bar, 128);
                }
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += CW) {
                    float o[CW];
                    load_tmem_cols<CW>(o_tmem + c0, o);
                    if (C::STAGE_O) {
                        // bf16 tile in the swizzled layout of the output tensor map
#pragma unroll
                        for (int g = 0; g < CW / 8; ++g) {
                            const int unit = (c0 + 8 * g) / 8;
                            const int ch = unit / (C::RB / 16);
                            const int u = unit % (C::RB / 16);
                            *reinterpret_cast<uint4*>(stage + ch * C::CHUNK_BYTES + swz_offset<C::RB>(row, u)) =
                                pack8_bf16(&o[8 * g], inv_l);
                        }
                    } else if (whole) {
                        if (row_valid) {
                            const size_t r = (MODE == kDecoderSample) ? static_cast<size_t>(it.out_row0 + prow)
                                                                      : static_cast<size_t>(it.q_z) * p.L + qrow;
                            uint4* dst = reinterpret_cast<uint4*>(outp + r * D + c0);
#pragma unroll
                            for (int c = 0; c < CW; c += 8) dst[c / 8] = pack8_bf16(&o[c], inv_l);
                        }
                    } else if (row_valid && prow < p.rows_cap) {
                        float4* so = reinterpret_cast<float4*>(slot + static_cast<size_t>(prow) * D + c0);
#pragma unroll
                        for (int c = 0; c < CW; c += 4) so[c / 4] = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
                    }
                }
                ptx::tc_fence_before();
                ptx::mbar_arrive(&o_free[ob * NQ + q]);

                if (MODE != kDecoderSample) {
                    if (C::STAGE_O) {
                        ptx::fence_proxy_async_smem();
                        ptx::named_barrier_sync(wg_bar, 128);
                        if (wtid == 0) {
                            for (int ch = 0; ch < C::NCH; ++ch)
                                ptx::tma_store_3d(&p.tm_o, stage + ch * C::CHUNK_BYTES, ch * (C::RB / 2),
                                                  it.q_row0 + q * kBlockM, it.q_z);
                            ptx::tma_store_commit();
                        }
                    }
                    if (p.lse != nullptr && row_valid) p.lse[static_cast<size_t>(it.q_z) * p.L + qrow] = lse_val;
                } else if (whole) {
                    if (p.lse != nullptr && row_valid) p.lse[it.out_row0 + prow] = lse_val;
                } else {
                    // Split unit: (O, m, l) of this CTA is in its slot; take a ticket; the last CTA
                    // of the unit merges every slot.
                    if (row_valid && prow < p.rows_cap) {
                        slot[p.rows_cap * D + prow] = m;
                        slot[p.rows_cap * D + p.rows_cap + prow] = l;
                    }
                    // Release: the barrier orders the warpgroup's slot stores before one thread's
                    // fence and ticket.
                    ptx::named_barrier_sync(wg_bar, 128);
                    if (wtid == 0) {
                        __threadfence();
                        const int ticket = atomicAdd(&p.ws_tickets[c_first], 1);
                        const int last = (ticket == c_last - c_first) ? 1 : 0;
                        if (last) p.ws_tickets[c_first] = 0;
                        *bcast = last;
                    }
                    ptx::named_barrier_sync(wg_bar, 128);
                    const int is_last = *bcast;
                    ptx::named_barrier_sync(wg_bar, 128);
                    if (is_last) {
                        __threadfence();
                        if (row_valid && prow < p.rows_cap) {
                            const long long T = it.total;
                            const int grid = it.sgrid;
                            auto slot_ptr = [&](int c) -> const float* {
                                const int si = (range_begin(c, T, grid) >= ubeg) ? 2 * c : 2 * c + 1;
                                return p.ws_partial + static_cast<size_t>(si) * p.slot_floats;
                            };
                            // Loads of different partials do not depend on each other: the loops are
                            // unrolled so that several L2 round trips overlap.
                            float mmax = -INFINITY;
#pragma unroll 4
                            for (int c = c_first; c <= c_last; ++c)
                                mmax = fmaxf(mmax, __ldcg(slot_ptr(c) + p.rows_cap * D + prow));
                            const float muse = (mmax == -INFINITY) ? 0.f : mmax;
                            float ltot = 0.f;
#pragma unroll 4
                            for (int c = c_first; c <= c_last; ++c) {
                                const float* sl = slot_ptr(c);
                                const float mw = __ldcg(sl + p.rows_cap * D + prow);
                                const float lw = __ldcg(sl + p.rows_cap * D + p.rows_cap + prow);
                                ltot += (mw == -INFINITY) ? 0.f : ptx::ex2(mw - muse) * lw;
                            }
                            const float inv = (ltot > 0.f) ? 1.f / ltot : 0.f;
                            uint4* dst = reinterpret_cast<uint4*>(outp + static_cast<size_t>(it.out_row0 + prow) * D);
#pragma unroll 1
                            for (int c0 = 0; c0 < D; c0 += CW) {
                                float acc[CW];
#pragma unroll
                                for (int c = 0; c < CW; ++c) acc[c] = 0.f;
#pragma unroll 2
                                for (int c = c_first; c <= c_last; ++c) {
                                    const float* sl = slot_ptr(c);
                                    const float mw = __ldcg(sl + p.rows_cap * D + prow);
                                    const float4* so = reinterpret_cast<const float4*>(sl + static_cast<size_t>(prow) * D + c0);
                                    float4 v[CW / 4];
#pragma unroll
                                    for (int c4 = 0; c4 < CW / 4; ++c4) v[c4] = __ldcg(so + c4);
                                    const float w = (mw == -INFINITY) ? 0.f : ptx::ex2(mw - muse);
#pragma unroll
                                    for (int c4 = 0; c4 < CW / 4; ++c4) {
                                        acc[4 * c4 + 0] += w * v[c4].x;
                                        acc[4 * c4 + 1] += w * v[c4].y;
                                        acc[4 * c4 + 2] += w * v[c4].z;
                                        acc[4 * c4 + 3] += w * v[c4].w;
                                    }
                                }
#pragma unroll
                                for (int c = 0; c < CW; c += 8) dst[(c0 + c) / 8] = pack8_bf16(&acc[c], inv);
                            }
                            if (p.lse != nullptr)
                                p.lse[it.out_row0 + prow] =
                                    (ltot > 0.f) ? (mmax + __log2f(ltot)) * 0.69314718055994531f : -INFINITY;
                        }
                    }
                }
                ++qitem;
            }
            if (C::STAGE_O && wtid == 0) ptx::tma_store_wait_all();
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(softmax_done);
    }

    // No common tail: each role returns on its own (warp 1 frees TMEM once softmax_done and
    // its own MMAs say nothing uses it any more).
#undef E2D2_SMEM_POINTERS
}

}  // namespace e2d2
