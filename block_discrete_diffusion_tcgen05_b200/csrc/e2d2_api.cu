// e2d2_api.cu -- host side of the C ABI declared in include/e2d2_attn.h: argument validation,
// TMA tensor-map encoding, grid choice and kernel launches on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <mutex>
#include <queue>
#include <utility>
#include <vector>

#include "attn_bwd_sm100.cuh"
#include "e2d2_attn.h"
#include "fmha_keyrow_sm100.cuh"
#include "fmha_sm100.cuh"
#include "kv_append.cuh"

namespace e2d2 {

__device__ unsigned int g_error_word = 0;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready = false;
    bool supported = false;
    int sms = 0;
    unsigned int* err = nullptr;
};

std::mutex g_mutex;
DeviceInfo g_dev[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

e2d2_status device_info(DeviceInfo** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return E2D2_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return E2D2_ERR_CUDA;
        d.supported = (prop.major == 10);
        d.sms = prop.multiProcessorCount;
        void* sym = nullptr;
        if (cudaGetSymbolAddress(&sym, g_error_word) != cudaSuccess) return E2D2_ERR_CUDA;
        d.err = static_cast<unsigned int*>(sym);
        if (!g_encode) {
            void* fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                    cudaSuccess ||
                q != cudaDriverEntryPointSuccess || fn == nullptr)
                return E2D2_ERR_CUDA;
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
        d.ready = true;
    }
    if (!d.supported) return E2D2_ERR_UNSUPPORTED;
    *out = &d;
    return E2D2_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

e2d2_status check_dims(const e2d2_dims& dm) {
    if (dm.batch <= 0 || dm.q_heads <= 0 || dm.kv_heads <= 0 || dm.head_dim <= 0)
        return E2D2_ERR_INVALID_ARG;
    if (dm.q_heads % dm.kv_heads != 0) return E2D2_ERR_INVALID_ARG;
    if (dm.head_dim != 32 && dm.head_dim != 64 && dm.head_dim != 128) return E2D2_ERR_UNSUPPORTED;
    if (!std::isfinite(dm.scale)) return E2D2_ERR_INVALID_ARG;
    return E2D2_OK;
}

float scale_log2(const e2d2_dims& dm) {
    const double s = dm.scale > 0.f ? static_cast<double>(dm.scale) : 1.0 / std::sqrt((double)dm.head_dim);
    return static_cast<float>(s * 1.4426950408889634);
}

// bf16 tensor [units][rows][D] (unit stride `unit_rows` rows), boxes of {min(D,64), box_rows, 1}.
bool map_3d(CUtensorMap* m, const void* base, int D, long long rows, long long units,
            long long unit_rows, int box_rows) {
    const int rb = (D * 2 < 128) ? D * 2 : 128;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                          static_cast<cuuint64_t>(units)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                             static_cast<cuuint64_t>(unit_rows) * D * 2};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(rb / 2), static_cast<cuuint32_t>(box_rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                                strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                rb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool map_2d(CUtensorMap* m, const void* base, int D, long long rows, int box_rows) {
    const int rb = (D * 2 < 128) ? D * 2 : 128;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(rb / 2), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                                strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                rb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Every kernel goes out with programmatic stream serialization: it may launch while the previous
// kernel on the stream is still running (its CTAs do their setup on free SMs) and waits for that
// kernel's completion (griddepcontrol.wait) before it reads or writes anything the caller owns.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

template <int D, int MODE>
e2d2_status launch_fmha(const FmhaParams& prm, int grid, cudaStream_t st,
                        const typename OrderOf<MODE>::type& ord = typename OrderOf<MODE>::type{}) {
    using SM = Smem<D, MODE>;
    static_assert(SM::ALLOC <= 232448, "shared memory budget");
    auto kern = fmha_sm100_kernel<D, MODE>;
    // Ask for at least ~116 KB so that two CTAs never share an SM (each takes all of TMEM).
    const int smem = SM::ALLOC > 118784 ? SM::ALLOC : 118784;
    static thread_local int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return E2D2_ERR_CUDA;
        configured_dev = dev;
    }
    return launch_pdl(kern, dim3(grid), dim3(kThreads), smem, st, prm, ord) == cudaSuccess ? E2D2_OK : E2D2_ERR_CUDA;
}

template <int N>
e2d2_status launch_keyrow(const FmhaParams& prm, int grid, cudaStream_t st) {
    using SM = KrSmem<N>;
    static_assert(SM::ALLOC <= 232448, "shared memory budget");
    auto kern = fmha_keyrow_kernel<N>;
    const int smem = SM::ALLOC > 118784 ? SM::ALLOC : 118784;
    static thread_local int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return E2D2_ERR_CUDA;
        configured_dev = dev;
    }
    return launch_pdl(kern, dim3(grid), dim3(kKrThreads), smem, st, prm) == cudaSuccess ? E2D2_OK : E2D2_ERR_CUDA;
}

template <int MODE>
e2d2_status dispatch_fmha(int D, const FmhaParams& prm, int grid, cudaStream_t st,
                          const typename OrderOf<MODE>::type& ord = typename OrderOf<MODE>::type{}) {
    switch (D) {
        case 32: return launch_fmha<32, MODE>(prm, grid, st, ord);
        case 64: return launch_fmha<64, MODE>(prm, grid, st, ord);
        case 128: return launch_fmha<128, MODE>(prm, grid, st, ord);
        default: return E2D2_ERR_UNSUPPORTED;
    }
}

// Work of train item k in tile steps: the key tiles of its stream (as the kernel's scheduler
// derives them), plus one for the epilogue and the next item's start.
int train_item_cost(int mode, int B, int Hq, int L, int S, int num_qtiles, int k) {
    const int BH = B * Hq;
    const int qp = num_qtiles - 1 - k / BH;
    const int r0 = qp * 2 * kBlockM;
    const int nact = (r0 + kBlockM < L) ? 2 : 1;
    int a1 = 1 << 30, e1 = 0, n0 = 0;
    for (int q = 0; q < nact; ++q) {
        const int rq = r0 + q * kBlockM;
        const int rl = (L < rq + kBlockM ? L : rq + kBlockM) - 1;
        const int blk_end = (rl / S + 1) * S < L ? (rl / S + 1) * S : L;
        int qa1, qe1, qn0;
        if (mode == kEncoder) {
            qa1 = 0;
            qe1 = 0;
            qn0 = (blk_end + kBlockN - 1) / kBlockN;
        } else {
            qa1 = ((rq / S) * S) / kBlockN;
            qe1 = (blk_end + kBlockN - 1) / kBlockN;
            qn0 = ((rl / S) * S + kBlockN - 1) / kBlockN;
        }
        if (qe1 > qa1) {
            a1 = a1 < qa1 ? a1 : qa1;
            e1 = e1 > qe1 ? e1 : qe1;
        }
        n0 = n0 > qn0 ? n0 : qn0;
    }
    if (e1 == 0) a1 = 0;
    return (e1 - a1) + n0 + 1;
}

// Longest processing time first: items by decreasing cost (ties by index), each to the CTA with
// the least work so far (ties by CTA index).  Fills `ord` (enabled = 0 if it does not fit).
// Cached per shape: the table is a pure function of it.
void train_item_order(int mode, int B, int Hq, int L, int S, int num_qtiles, int num_items, int grid, ItemOrder* ord) {
    ord->enabled = 0;
    if (num_items > kOrderMaxItems || grid > kOrderMaxCtas || grid <= 0) return;
    struct Key {
        int mode, B, Hq, L, S, grid;
        bool operator==(const Key& o) const {
            return mode == o.mode && B == o.B && Hq == o.Hq && L == o.L && S == o.S && grid == o.grid;
        }
    };
    struct Entry {
        Key key;
        ItemOrder ord;
    };
    static std::mutex mu;
    static std::vector<Entry> cache;  // a few shapes; oldest dropped first
    const Key key{mode, B, Hq, L, S, grid};
    {
        std::lock_guard<std::mutex> lock(mu);
        for (const Entry& e : cache)
            if (e.key == key) {
                *ord = e.ord;
                return;
            }
    }
    std::vector<int> cost(num_items), idx(num_items);
    for (int k = 0; k < num_items; ++k) {
        cost[k] = train_item_cost(mode, B, Hq, L, S, num_qtiles, k);
        idx[k] = k;
    }
    std::stable_sort(idx.begin(), idx.end(), [&](int a, int b) { return cost[a] > cost[b]; });
    using Load = std::pair<long long, int>;  // (work so far, CTA)
    std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
    for (int c = 0; c < grid; ++c) heap.push({0, c});
    std::vector<std::vector<int>> per(grid);
    for (int k : idx) {
        Load t = heap.top();
        heap.pop();
        per[t.second].push_back(k);
        t.first += cost[k];
        heap.push(t);
    }
    int pos = 0;
    for (int c = 0; c < grid; ++c) {
        ord->first[c] = static_cast<uint16_t>(pos);
        for (int k : per[c]) ord->item[pos++] = static_cast<uint16_t>(k);
    }
    ord->first[grid] = static_cast<uint16_t>(pos);
    ord->enabled = 1;
    std::lock_guard<std::mutex> lock(mu);
    if (cache.size() >= 8) cache.erase(cache.begin());
    cache.push_back({key, *ord});
}

constexpr long long kMaxI32 = 0x7fffffffLL;

e2d2_status check_train_shape(const e2d2_dims& dm, int L, int S) {
    // S need not divide L: the last block then has L mod S rows; S >= L is one block.
    if (L <= 0 || S <= 0) return E2D2_ERR_INVALID_ARG;
    const long long rows = static_cast<long long>(dm.batch) * dm.q_heads * L;
    if (rows > kMaxI32 / 8) return E2D2_ERR_SHAPE;
    return E2D2_OK;
}

e2d2_status train_common(int mode, const void* q, const void* k0, const void* v0, const void* k1,
                         const void* v1, void* out, float* lse, const e2d2_dims& dm, int L, int S,
                         cudaStream_t st) {
    e2d2_status s = check_dims(dm);
    if (s != E2D2_OK) return s;
    s = check_train_shape(dm, L, S);
    if (s != E2D2_OK) return s;
    if (!aligned16(q) || !aligned16(k0) || !aligned16(v0) || !aligned16(out) ||
        (k1 && !aligned16(k1)) || (v1 && !aligned16(v1)) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
        return E2D2_ERR_ALIGNMENT;
    DeviceInfo* di = nullptr;
    s = device_info(&di);
    if (s != E2D2_OK) return s;

    const int D = dm.head_dim;
    FmhaParams prm;
    std::memset(&prm, 0, sizeof(prm));
    const long long BHq = static_cast<long long>(dm.batch) * dm.q_heads;
    const long long BHkv = static_cast<long long>(dm.batch) * dm.kv_heads;
    bool ok = map_3d(&prm.tm_q, q, D, L, BHq, L, kBlockM) && map_3d(&prm.tm_o, out, D, L, BHq, L, kBlockM) &&
              map_3d(&prm.tm_k0, k0, D, L, BHkv, L, kBlockN) && map_3d(&prm.tm_v0, v0, D, L, BHkv, L, kBlockN);
    if (mode == kDecoderTrain)
        ok = ok && map_3d(&prm.tm_k1, k1, D, L, BHkv, L, kBlockN) && map_3d(&prm.tm_v1, v1, D, L, BHkv, L, kBlockN);
    if (!ok) return E2D2_ERR_CUDA;
    prm.out = out;
    prm.lse = lse;
    prm.err = di->err;
    prm.batch = dm.batch;
    prm.q_heads = dm.q_heads;
    prm.kv_heads = dm.kv_heads;
    prm.group = dm.q_heads / dm.kv_heads;
    prm.L = L;
    prm.S = S;
    prm.box1_rows = kBlockN;
    prm.scale_log2 = scale_log2(dm);
    prm.num_qtiles = (L + 2 * kBlockM - 1) / (2 * kBlockM);  // work items take pairs of query tiles
    prm.num_items = static_cast<int>(BHq * prm.num_qtiles);
    const int grid = prm.num_items < di->sms ? prm.num_items : di->sms;
    ItemOrder ord;
    train_item_order(mode, dm.batch, dm.q_heads, L, S, prm.num_qtiles, prm.num_items, grid, &ord);
    return mode == kEncoder ? dispatch_fmha<kEncoder>(D, prm, grid, st, ord)
                            : dispatch_fmha<kDecoderTrain>(D, prm, grid, st, ord);
}

// Backward of the train calls: two launches of attn_bwd_sm100_kernel on the stream, rows-Q
// (dq, and D_i / -lse_i log2e into the workspace), then rows-KV (dk, dv).
struct BwdArgs {
    const void *q, *k0, *v0, *k1, *v1, *out, *dout;
    const float* lse;
    void *dq, *dk0, *dv0, *dk1, *dv1;
};

long long bwd_lpad(int L) { return (static_cast<long long>(L) + kBwdRows - 1) / kBwdRows * kBwdRows; }

template <int D, int SIDE>
e2d2_status launch_bwd(const BwdTcParams& prm, int grid, cudaStream_t st) {
    using SM = BwdSmem<D>;
    static_assert(SM::ALLOC <= 232448, "shared memory budget");
    auto kern = attn_bwd_sm100_kernel<D, SIDE>;
    const int smem = SM::ALLOC > 118784 ? SM::ALLOC : 118784;
    static thread_local int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return E2D2_ERR_CUDA;
        configured_dev = dev;
    }
    return launch_pdl(kern, dim3(grid), dim3(kThreads), smem, st, prm) == cudaSuccess ? E2D2_OK : E2D2_ERR_CUDA;
}

template <int SIDE>
e2d2_status dispatch_bwd(int D, const BwdTcParams& prm, int grid, cudaStream_t st) {
    switch (D) {
        case 32: return launch_bwd<32, SIDE>(prm, grid, st);
        case 64: return launch_bwd<64, SIDE>(prm, grid, st);
        case 128: return launch_bwd<128, SIDE>(prm, grid, st);
        default: return E2D2_ERR_UNSUPPORTED;
    }
}

e2d2_status train_backward(bool decoder, const BwdArgs& a, const e2d2_dims& dm, int L, int S, void* workspace,
                           size_t ws_bytes, cudaStream_t st) {
    e2d2_status s = check_dims(dm);
    if (s != E2D2_OK) return s;
    s = check_train_shape(dm, L, S);
    if (s != E2D2_OK) return s;
    const long long Lpad = bwd_lpad(L);
    const size_t need = 2 * static_cast<size_t>(dm.batch) * dm.q_heads * Lpad * sizeof(float);
    if (!workspace || ws_bytes < need) return E2D2_ERR_WORKSPACE;
    const void* ptrs[] = {a.q, a.k0, a.v0, a.out, a.dout, a.dq, a.dk0, a.dv0, workspace};
    for (const void* ptr : ptrs)
        if (!aligned16(ptr)) return E2D2_ERR_ALIGNMENT;
    if (decoder && (!aligned16(a.k1) || !aligned16(a.v1) || !aligned16(a.dk1) || !aligned16(a.dv1)))
        return E2D2_ERR_ALIGNMENT;
    if (reinterpret_cast<uintptr_t>(a.lse) & 3u) return E2D2_ERR_ALIGNMENT;
    DeviceInfo* di = nullptr;
    s = device_info(&di);
    if (s != E2D2_OK) return s;

    const int D = dm.head_dim;
    const long long BHq = static_cast<long long>(dm.batch) * dm.q_heads;
    const long long BHkv = static_cast<long long>(dm.batch) * dm.kv_heads;
    BwdTcParams prm;
    std::memset(&prm, 0, sizeof(prm));
    prm.lse = a.lse;
    prm.out = static_cast<const __nv_bfloat16*>(a.out);
    prm.dout = static_cast<const __nv_bfloat16*>(a.dout);
    prm.ws_nl2 = static_cast<float*>(workspace);
    prm.ws_D = static_cast<float*>(workspace) + BHq * Lpad;
    prm.err = di->err;
    prm.batch = dm.batch;
    prm.q_heads = dm.q_heads;
    prm.kv_heads = dm.kv_heads;
    prm.group = dm.q_heads / dm.kv_heads;
    prm.L = L;
    prm.S = S;
    prm.Lpad = static_cast<int>(Lpad);
    prm.decoder = decoder ? 1 : 0;
    prm.scale = static_cast<float>(dm.scale > 0.f ? static_cast<double>(dm.scale)
                                                  : 1.0 / std::sqrt(static_cast<double>(dm.head_dim)));
    prm.scale_log2 = scale_log2(dm);
    prm.n_row_tiles = (L + kBwdRows - 1) / kBwdRows;
    const void* k1 = decoder ? a.k1 : a.k0;
    const void* v1 = decoder ? a.v1 : a.v0;

    // rows-Q: row tiles Q, dO (128 rows); column sub-tiles K, V of each key source (64 rows).
    BwdTcParams pq = prm;
    bool ok = map_3d(&pq.tm_r1[0], a.q, D, L, BHq, L, kBwdRows) && map_3d(&pq.tm_r2[0], a.dout, D, L, BHq, L, kBwdRows) &&
              map_3d(&pq.tm_c1[0], a.k0, D, L, BHkv, L, kBwdCols) && map_3d(&pq.tm_c2[0], a.v0, D, L, BHkv, L, kBwdCols) &&
              map_3d(&pq.tm_c1[1], k1, D, L, BHkv, L, kBwdCols) && map_3d(&pq.tm_c2[1], v1, D, L, BHkv, L, kBwdCols);
    ok = ok && map_3d(&pq.tm_ga[0], a.dq, D, L, BHq, L, kBwdRows) && map_3d(&pq.tm_out, a.out, D, L, BHq, L, kBwdRows);
    pq.tm_ga[1] = pq.tm_gb[0] = pq.tm_gb[1] = pq.tm_ga[0];
    pq.tm_r1[1] = pq.tm_r1[0];
    pq.tm_r2[1] = pq.tm_r2[0];
    pq.g_a[0] = pq.g_a[1] = static_cast<__nv_bfloat16*>(a.dq);
    pq.num_items = static_cast<int>(BHq * prm.n_row_tiles);
    // rows-KV: row tiles K, V of each key source (128 rows); column sub-tiles Q, dO (64 rows).
    BwdTcParams pk = prm;
    ok = ok && map_3d(&pk.tm_r1[0], a.k0, D, L, BHkv, L, kBwdRows) && map_3d(&pk.tm_r2[0], a.v0, D, L, BHkv, L, kBwdRows) &&
         map_3d(&pk.tm_r1[1], k1, D, L, BHkv, L, kBwdRows) && map_3d(&pk.tm_r2[1], v1, D, L, BHkv, L, kBwdRows) &&
         map_3d(&pk.tm_c1[0], a.q, D, L, BHq, L, kBwdCols) && map_3d(&pk.tm_c2[0], a.dout, D, L, BHq, L, kBwdCols) &&
         map_3d(&pk.tm_ga[0], a.dv0, D, L, BHkv, L, kBwdRows) && map_3d(&pk.tm_gb[0], a.dk0, D, L, BHkv, L, kBwdRows) &&
         map_3d(&pk.tm_ga[1], decoder ? a.dv1 : a.dv0, D, L, BHkv, L, kBwdRows) &&
         map_3d(&pk.tm_gb[1], decoder ? a.dk1 : a.dk0, D, L, BHkv, L, kBwdRows);
    if (!ok) return E2D2_ERR_CUDA;
    pk.tm_c1[1] = pk.tm_c1[0];
    pk.tm_c2[1] = pk.tm_c2[0];
    pk.tm_out = pk.tm_ga[0];  // unused on this side
    pk.g_a[0] = static_cast<__nv_bfloat16*>(a.dv0);
    pk.g_b[0] = static_cast<__nv_bfloat16*>(a.dk0);
    pk.g_a[1] = static_cast<__nv_bfloat16*>(decoder ? a.dv1 : a.dv0);
    pk.g_b[1] = static_cast<__nv_bfloat16*>(decoder ? a.dk1 : a.dk0);
    pk.num_items = static_cast<int>((decoder ? 2 : 1) * BHkv * prm.n_row_tiles);

    const int gq = pq.num_items < di->sms ? pq.num_items : di->sms;
    const int gk = pk.num_items < di->sms ? pk.num_items : di->sms;
    s = dispatch_bwd<kBwdRowsQ>(D, pq, gq, st);
    if (s != E2D2_OK) return s;
    return dispatch_bwd<kBwdRowsKV>(D, pk, gk, st);
}

struct SampleLayout {
    int rows_cap;
    int slot_floats;
    size_t bytes;
};

SampleLayout sample_layout(const e2d2_dims& dm, int S) {
    SampleLayout w;
    const long long rows = static_cast<long long>(dm.q_heads / dm.kv_heads) * S;
    w.rows_cap = static_cast<int>(rows < kBlockM ? rows : kBlockM);
    const long long f = static_cast<long long>(w.rows_cap) * (dm.head_dim + 2);
    w.slot_floats = static_cast<int>((f + 63) / 64 * 64);
    w.bytes = 1024 + static_cast<size_t>(2) * kSampleMaxCtas * w.slot_floats * sizeof(float);
    return w;
}

// Work plan of a sampling call: which kernel, how many units and key tiles, and the two-phase
// split.  With U units on G CTAs, floor(U/G)*G units run whole (one CTA each, last); the other R
// units are split stream-K over at most 5R CTAs (a unit has at most about six partials to merge),
// and only as far as every piece keeps about kMinSplitTiles key tiles: publishing and merging a
// partial costs several microseconds, more than streaming a few tiles.  A split never uses fewer
// CTAs than there are units, so a CTA's tile range meets at most two units (two partial slots).
struct SamplePlan {
    int keyrow_n;        // 0: generic kernel; 16/32/64: keys-on-lanes kernel with N query columns
    int num_qtiles;      // query tiles per (batch, kv head)
    int tiles_per_unit;  // 128-key tiles per unit: prefix tiles + own-block tiles
    int split_units;     // R
    int whole_units;     // U - R
    int split_ctas;      // CTAs of the split phase
    long long total_tiles;  // key tiles of the split phase (R * tiles_per_unit)
    long long grid;      // CTAs launched
};

// E2D2_SPLITS=n (read once per process): CTAs of the split phase, for tests of split-count
// independence; clamped to what the schedule supports.  0 or unset: the heuristic below.
int split_override() {
    static const int v = [] {
        const char* e = std::getenv("E2D2_SPLITS");
        return e ? std::atoi(e) : 0;
    }();
    return v;
}

SamplePlan plan_sample(const e2d2_dims& dims, int S, int P, int sms) {
    SamplePlan pl;
    const int D = dims.head_dim;
    const int G = dims.q_heads / dims.kv_heads;
    const long long BHkv = static_cast<long long>(dims.batch) * dims.kv_heads;
    // Short packed tiles at d = 128 take the kernel with keys on the TMEM lanes (S^T = K Q^T):
    // its tensor-core rows are keys, so none is padding.  N = packed columns rounded up.
    const int GS = G * S;
    pl.keyrow_n = (D != 128 || GS > 64) ? 0 : (GS <= 16 ? 16 : (GS <= 32 ? 32 : 64));
    pl.num_qtiles = pl.keyrow_n ? 1 : (G * S + kBlockM - 1) / kBlockM;
    pl.tiles_per_unit = (S + kBlockN - 1) / kBlockN + (P + kBlockN - 1) / kBlockN;
    const long long Tu = pl.tiles_per_unit;
    const long long U = BHkv * pl.num_qtiles;
    long long grid = sms < kSampleMaxCtas ? sms : kSampleMaxCtas;
    if (grid > U * Tu) grid = U * Tu;
    const long long R = U >= grid ? U % grid : U;
    pl.split_units = static_cast<int>(R);
    pl.whole_units = static_cast<int>(U - R);
    constexpr long long kMinSplitTiles = 6;
    long long sc = R * 5 < grid ? R * 5 : grid;
    if (sc > R * Tu / kMinSplitTiles) sc = R * Tu / kMinSplitTiles;
    if (sc < R) sc = R;
    if (split_override() > 0 && R > 0) sc = split_override() < grid ? split_override() : grid;
    if (sc < R) sc = R;
    if (sc > R * Tu) sc = R * Tu;
    pl.split_ctas = static_cast<int>(sc);
    pl.total_tiles = R * Tu;
    // Whole units exist only when U >= grid, and then every CTA takes some; otherwise only the
    // CTAs of the split phase have work.
    if (pl.whole_units == 0) grid = pl.split_ctas;
    pl.grid = grid;
    return pl;
}

// A sampling call, checked and encoded but not yet launched.
struct SampleLaunch {
    FmhaParams prm;
    int keyrow_n;
    int head_dim;
    long long grid;
};

// Every check of a sampling call and the kernel parameters; launches and enqueues nothing, so an
// error return leaves the stream untouched.  `append` (encoder block step) also writes the block's
// K/V to cache rows P..P+S-1 from inside the same launch.
e2d2_status sample_prepare(bool append, const void* q_blk, const void* k_cache, const void* v_cache, int capacity,
                           int P, const int* P_dev, const void* k_blk, const void* v_blk, void* out, float* lse,
                           e2d2_dims dims, int S, void* workspace, size_t ws_bytes, SampleLaunch* sl) {
    if (!q_blk || !k_cache || !v_cache || !k_blk || !v_blk || !out) return E2D2_ERR_INVALID_ARG;
    e2d2_status s = check_dims(dims);
    if (s != E2D2_OK) return s;
    if (S <= 0 || capacity < 0 || P < 0) return E2D2_ERR_INVALID_ARG;
    if (P > capacity || (append && static_cast<long long>(P) + S > capacity)) return E2D2_ERR_CAPACITY;
    const long long rows = static_cast<long long>(dims.batch) * dims.q_heads * S;
    if (rows > kMaxI32 / 8 || static_cast<long long>(capacity) * dims.batch * dims.kv_heads > kMaxI32)
        return E2D2_ERR_SHAPE;
    if (P_dev != nullptr) {
        if (reinterpret_cast<uintptr_t>(P_dev) & 3u) return E2D2_ERR_ALIGNMENT;
        if (dims.batch > kRaggedMaxBatch) return E2D2_ERR_SHAPE;
        // every tile index of the stream fits in an int
        const long long units = static_cast<long long>(dims.batch) * dims.kv_heads *
                                ((static_cast<long long>(dims.q_heads / dims.kv_heads) * S + kBlockM - 1) / kBlockM);
        if (units * ((capacity + kBlockN - 1) / kBlockN + (S + kBlockN - 1) / kBlockN) > kMaxI32) return E2D2_ERR_SHAPE;
    }
    if (!aligned16(q_blk) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_blk) ||
        !aligned16(v_blk) || !aligned16(out) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
        return E2D2_ERR_ALIGNMENT;
    const SampleLayout w = sample_layout(dims, S);
    if (!workspace || ws_bytes < w.bytes) return E2D2_ERR_WORKSPACE;
    if (!aligned16(workspace)) return E2D2_ERR_ALIGNMENT;
    DeviceInfo* di = nullptr;
    s = device_info(&di);
    if (s != E2D2_OK) return s;

    const int D = dims.head_dim;
    const int G = dims.q_heads / dims.kv_heads;
    FmhaParams& prm = sl->prm;
    std::memset(&prm, 0, sizeof(prm));
    const long long BHkv = static_cast<long long>(dims.batch) * dims.kv_heads;
    const int S16 = (S + 15) / 16 * 16;
    const int box1 = S16 < kBlockN ? S16 : kBlockN;
    // Packed query rows per TMEM lane quarter.  The kernel can spread a short packed tile over the
    // four lane quarters (q_chunk < 32); on B200 that measured slower for the sampling shapes (four
    // warps then issue full-width TMEM loads and instruction streams for a quarter of the rows
    // each), so rows stay contiguous.
    const int q_chunk = kBlockM / 4;
    const SamplePlan plan = plan_sample(dims, S, P, di->sms);
    const int keyrow_n = plan.keyrow_n;
    // Single prefix: cache rows >= P lie outside the map (zeros, never read).  Ragged prefixes: the
    // map spans the capacity; the kernels mask keys past each entry's P and zero those V rows.
    const int map_rows = P_dev != nullptr ? capacity : P;
    bool ok = map_2d(&prm.tm_q, q_blk, D, rows, keyrow_n ? keyrow_n : q_chunk) &&
              map_3d(&prm.tm_k0, k_cache, D, map_rows > 0 ? map_rows : 1, BHkv, capacity > 0 ? capacity : 1, kBlockN) &&
              map_3d(&prm.tm_v0, v_cache, D, map_rows > 0 ? map_rows : 1, BHkv, capacity > 0 ? capacity : 1, kBlockN) &&
              map_3d(&prm.tm_k1, k_blk, D, S, BHkv, S, box1) && map_3d(&prm.tm_v1, v_blk, D, S, BHkv, S, box1);
    if (!ok) return E2D2_ERR_CUDA;
    prm.out = out;
    prm.lse = lse;
    prm.ws_tickets = static_cast<int*>(workspace);
    prm.ws_partial = reinterpret_cast<float*>(static_cast<char*>(workspace) + 1024);
    prm.err = di->err;
    prm.batch = dims.batch;
    prm.q_heads = dims.q_heads;
    prm.kv_heads = dims.kv_heads;
    prm.group = G;
    prm.L = S;
    prm.S = S;
    prm.P = P;
    prm.box1_rows = box1;
    prm.scale_log2 = scale_log2(dims);
    prm.rows_per_unit = G * S;
    prm.num_qtiles = plan.num_qtiles;
    prm.tiles_per_unit = plan.tiles_per_unit;
    prm.rows_cap = w.rows_cap;
    prm.q_chunk = q_chunk;
    prm.slot_floats = w.slot_floats;
    if (append) {
        prm.app_src_k = static_cast<const uint4*>(k_blk);
        prm.app_src_v = static_cast<const uint4*>(v_blk);
        prm.app_dst_k = static_cast<uint4*>(const_cast<void*>(k_cache));
        prm.app_dst_v = static_cast<uint4*>(const_cast<void*>(v_cache));
        prm.app_capacity = capacity;
    }
    prm.split_units = plan.split_units;
    prm.whole_units = plan.whole_units;
    prm.split_ctas = plan.split_ctas;
    prm.total_tiles = plan.total_tiles;
    sl->keyrow_n = keyrow_n;
    sl->head_dim = D;
    sl->grid = plan.grid;
    if (P_dev != nullptr) {
        // one stream-K stream over every unit's tiles, cut over a full grid (the tile count is
        // known only on the device)
        const int grid = di->sms < kSampleMaxCtas ? di->sms : kSampleMaxCtas;
        prm.P_dev = P_dev;
        prm.rg_capacity = capacity;
        prm.rg_units_per_entry = dims.kv_heads * plan.num_qtiles;
        prm.split_units = prm.whole_units = 0;
        prm.total_tiles = 0;
        prm.split_ctas = grid;
        sl->grid = grid;
    }
    return E2D2_OK;
}

e2d2_status sample_launch(const SampleLaunch& sl, cudaStream_t stream) {
    const int grid = static_cast<int>(sl.grid);
    switch (sl.keyrow_n) {
        case 16: return launch_keyrow<16>(sl.prm, grid, stream);
        case 32: return launch_keyrow<32>(sl.prm, grid, stream);
        case 64: return launch_keyrow<64>(sl.prm, grid, stream);
        default: return dispatch_fmha<kDecoderSample>(sl.head_dim, sl.prm, grid, stream);
    }
}

e2d2_status sample_call(bool append, const void* q_blk, const void* k_cache, const void* v_cache, int capacity,
                        int P, const void* k_blk, const void* v_blk, void* out, float* lse, e2d2_dims dims, int S,
                        void* workspace, size_t ws_bytes, cudaStream_t stream) {
    SampleLaunch sl;
    const e2d2_status s = sample_prepare(append, q_blk, k_cache, v_cache, capacity, P, nullptr, k_blk, v_blk, out, lse,
                                         dims, S, workspace, ws_bytes, &sl);
    return s != E2D2_OK ? s : sample_launch(sl, stream);
}

}  // namespace
}  // namespace e2d2

using namespace e2d2;

extern "C" {

const char* e2d2_status_string(e2d2_status s) {
    switch (s) {
        case E2D2_OK: return "E2D2_OK";
        case E2D2_ERR_INVALID_ARG: return "E2D2_ERR_INVALID_ARG";
        case E2D2_ERR_UNSUPPORTED: return "E2D2_ERR_UNSUPPORTED";
        case E2D2_ERR_SHAPE: return "E2D2_ERR_SHAPE";
        case E2D2_ERR_ALIGNMENT: return "E2D2_ERR_ALIGNMENT";
        case E2D2_ERR_CAPACITY: return "E2D2_ERR_CAPACITY";
        case E2D2_ERR_WORKSPACE: return "E2D2_ERR_WORKSPACE";
        case E2D2_ERR_CUDA: return "E2D2_ERR_CUDA";
        case E2D2_ERR_TIMEOUT: return "E2D2_ERR_TIMEOUT";
        case E2D2_ERR_DEVICE_CHECK: return "E2D2_ERR_DEVICE_CHECK";
    }
    return "E2D2_ERR_UNKNOWN";
}

int e2d2_version(void) { return 100; }

e2d2_status e2d2_attn_encoder_blockcausal(const void* q, const void* k, const void* v, void* out,
                                          float* lse, e2d2_dims dims, int L, int S,
                                          cudaStream_t stream) {
    if (!q || !k || !v || !out) return E2D2_ERR_INVALID_ARG;
    return train_common(kEncoder, q, k, v, nullptr, nullptr, out, lse, dims, L, S, stream);
}

e2d2_status e2d2_attn_decoder_train(const void* q_dec, const void* k_enc, const void* v_enc,
                                    const void* k_dec, const void* v_dec, void* out, float* lse,
                                    e2d2_dims dims, int L, int S, cudaStream_t stream) {
    if (!q_dec || !k_enc || !v_enc || !k_dec || !v_dec || !out) return E2D2_ERR_INVALID_ARG;
    return train_common(kDecoderTrain, q_dec, k_enc, v_enc, k_dec, v_dec, out, lse, dims, L, S, stream);
}

size_t e2d2_attn_train_backward_workspace(e2d2_dims dims, int L) {
    if (check_dims(dims) != E2D2_OK || L <= 0) return 0;
    return 2 * static_cast<size_t>(dims.batch) * dims.q_heads * bwd_lpad(L) * sizeof(float);
}

e2d2_status e2d2_attn_encoder_backward(const void* q, const void* k, const void* v, const void* out,
                                       const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                       e2d2_dims dims, int L, int S, void* workspace, size_t ws_bytes,
                                       cudaStream_t stream) {
    if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv) return E2D2_ERR_INVALID_ARG;
    BwdArgs a;
    std::memset(&a, 0, sizeof(a));
    a.q = q;
    a.k0 = k;
    a.v0 = v;
    a.out = out;
    a.lse = lse;
    a.dout = dout;
    a.dq = dq;
    a.dk0 = dk;
    a.dv0 = dv;
    return train_backward(false, a, dims, L, S, workspace, ws_bytes, stream);
}

e2d2_status e2d2_attn_decoder_train_backward(const void* q_dec, const void* k_enc, const void* v_enc,
                                             const void* k_dec, const void* v_dec, const void* out,
                                             const float* lse, const void* dout, void* dq, void* dk_enc,
                                             void* dv_enc, void* dk_dec, void* dv_dec, e2d2_dims dims, int L,
                                             int S, void* workspace, size_t ws_bytes, cudaStream_t stream) {
    if (!q_dec || !k_enc || !v_enc || !k_dec || !v_dec || !out || !lse || !dout || !dq || !dk_enc ||
        !dv_enc || !dk_dec || !dv_dec)
        return E2D2_ERR_INVALID_ARG;
    BwdArgs a;
    std::memset(&a, 0, sizeof(a));
    a.q = q_dec;
    a.k0 = k_enc;
    a.v0 = v_enc;
    a.k1 = k_dec;
    a.v1 = v_dec;
    a.out = out;
    a.lse = lse;
    a.dout = dout;
    a.dq = dq;
    a.dk0 = dk_enc;
    a.dv0 = dv_enc;
    a.dk1 = dk_dec;
    a.dv1 = dv_dec;
    return train_backward(true, a, dims, L, S, workspace, ws_bytes, stream);
}

size_t e2d2_attn_decoder_sample_workspace(e2d2_dims dims, int S, int capacity) {
    if (check_dims(dims) != E2D2_OK || S <= 0 || capacity < 0) return 0;
    return sample_layout(dims, S).bytes;
}

e2d2_status e2d2_attn_decoder_sample_plan(e2d2_dims dims, int S, int P, int num_sms, e2d2_sample_plan* plan) {
    if (!plan) return E2D2_ERR_INVALID_ARG;
    e2d2_status s = check_dims(dims);
    if (s != E2D2_OK) return s;
    if (S <= 0 || P < 0 || num_sms <= 0) return E2D2_ERR_INVALID_ARG;
    const SamplePlan pl = plan_sample(dims, S, P, num_sms);
    plan->kernel = pl.keyrow_n;
    plan->units = static_cast<int>(static_cast<long long>(dims.batch) * dims.kv_heads * pl.num_qtiles);
    plan->tiles_per_unit = pl.tiles_per_unit;
    plan->split_units = pl.split_units;
    plan->split_ctas = pl.split_ctas;
    plan->whole_units = pl.whole_units;
    plan->grid = static_cast<int>(pl.grid);
    return E2D2_OK;
}

e2d2_status e2d2_attn_train_order(int decoder, e2d2_dims dims, int L, int S, int num_sms, int* cta_of_item,
                                  int* items_out, int* grid_out, int* balanced_out) {
    e2d2_status s = check_dims(dims);
    if (s != E2D2_OK) return s;
    if (L <= 0 || S <= 0 || num_sms <= 0) return E2D2_ERR_INVALID_ARG;
    s = check_train_shape(dims, L, S);
    if (s != E2D2_OK) return s;
    const int mode = decoder ? kDecoderTrain : kEncoder;
    const int num_qtiles = (L + 2 * kBlockM - 1) / (2 * kBlockM);
    const long long items = static_cast<long long>(dims.batch) * dims.q_heads * num_qtiles;
    const int grid = static_cast<int>(items < num_sms ? items : num_sms);
    ItemOrder ord;
    train_item_order(mode, dims.batch, dims.q_heads, L, S, num_qtiles, static_cast<int>(items), grid, &ord);
    if (cta_of_item) {
        if (ord.enabled) {
            for (int c = 0; c < grid; ++c)
                for (int j = ord.first[c]; j < ord.first[c + 1]; ++j) cta_of_item[ord.item[j]] = c;
        } else {
            for (long long k = 0; k < items; ++k) cta_of_item[k] = static_cast<int>(k % grid);
        }
    }
    if (items_out) *items_out = static_cast<int>(items);
    if (grid_out) *grid_out = grid;
    if (balanced_out) *balanced_out = ord.enabled;
    return E2D2_OK;
}

e2d2_status e2d2_attn_decoder_sample(const void* q_blk, const void* k_cache, const void* v_cache,
                                     int capacity, int P, const void* k_blk, const void* v_blk,
                                     void* out, float* lse, e2d2_dims dims, int S, void* workspace,
                                     size_t ws_bytes, cudaStream_t stream) {
    return sample_call(false, q_blk, k_cache, v_cache, capacity, P, k_blk, v_blk, out, lse, dims, S, workspace,
                       ws_bytes, stream);
}

e2d2_status e2d2_attn_encoder_block_step(const void* q_blk, void* k_cache, void* v_cache, int capacity, int P,
                                         const void* k_blk, const void* v_blk, void* out, float* lse,
                                         e2d2_dims dims, int S, void* workspace, size_t ws_bytes,
                                         cudaStream_t stream) {
    return sample_call(true, q_blk, k_cache, v_cache, capacity, P, k_blk, v_blk, out, lse, dims, S, workspace,
                       ws_bytes, stream);
}

e2d2_status e2d2_attn_decoder_sample_ragged(const void* q_blk, const void* k_cache, const void* v_cache, int capacity,
                                            const int* P_dev, const void* k_blk, const void* v_blk, void* out,
                                            float* lse, e2d2_dims dims, int S, void* workspace, size_t ws_bytes,
                                            cudaStream_t stream) {
    if (!P_dev) return E2D2_ERR_INVALID_ARG;
    SampleLaunch sl;
    const e2d2_status s = sample_prepare(false, q_blk, k_cache, v_cache, capacity, 0, P_dev, k_blk, v_blk, out, lse,
                                         dims, S, workspace, ws_bytes, &sl);
    return s != E2D2_OK ? s : sample_launch(sl, stream);
}

e2d2_status e2d2_attn_decoder_sample_ragged_plan(e2d2_dims dims, int S, const int* P_host, int capacity, int num_sms,
                                                 e2d2_ragged_plan* plan) {
    if (!plan || !P_host) return E2D2_ERR_INVALID_ARG;
    e2d2_status s = check_dims(dims);
    if (s != E2D2_OK) return s;
    if (S <= 0 || capacity < 0 || num_sms <= 0) return E2D2_ERR_INVALID_ARG;
    if (dims.batch > kRaggedMaxBatch) return E2D2_ERR_SHAPE;
    const SamplePlan pl = plan_sample(dims, S, 0, num_sms);
    const int upe = dims.kv_heads * pl.num_qtiles;
    long long total = 0;
    for (int b = 0; b < dims.batch; ++b) total += ragged_entry_tiles(ragged_clamp(P_host[b], capacity), S, upe);
    plan->kernel = pl.keyrow_n;
    plan->units = dims.batch * upe;
    plan->units_per_entry = upe;
    plan->total_tiles = total;
    plan->grid = num_sms < kSampleMaxCtas ? num_sms : kSampleMaxCtas;
    long long g = total / kMinRaggedTiles;
    if (g < plan->units) g = plan->units;
    if (g > plan->grid) g = plan->grid;
    if (g > total) g = total;
    plan->stream_ctas = static_cast<int>(g);
    return E2D2_OK;
}

namespace {
e2d2_status append_call(void* k_cache, void* v_cache, int capacity, int P, const int* P_dev, const void* k_new,
                        const void* v_new, int S_new, const e2d2_dims& dims, cudaStream_t stream) {
    if (!k_cache || !v_cache || !k_new || !v_new) return E2D2_ERR_INVALID_ARG;
    e2d2_status s = check_dims(dims);
    if (s != E2D2_OK) return s;
    if (P < 0 || S_new < 0 || capacity < 0) return E2D2_ERR_INVALID_ARG;
    if (static_cast<long long>(P) + S_new > capacity) return E2D2_ERR_CAPACITY;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_new) || !aligned16(v_new) ||
        (reinterpret_cast<uintptr_t>(P_dev) & 3u))
        return E2D2_ERR_ALIGNMENT;
    if (S_new == 0) return E2D2_OK;
    DeviceInfo* di = nullptr;
    s = device_info(&di);
    if (s != E2D2_OK) return s;
    AppendParams a;
    a.cache[0] = static_cast<uint4*>(k_cache);
    a.cache[1] = static_cast<uint4*>(v_cache);
    a.src[0] = static_cast<const uint4*>(k_new);
    a.src[1] = static_cast<const uint4*>(v_new);
    a.capacity = capacity;
    a.P = P;
    a.S_new = S_new;
    a.vec_per_row = dims.head_dim / 8;
    a.units = dims.batch * dims.kv_heads;
    a.P_dev = P_dev;
    a.kv_heads = dims.kv_heads;
    const long long total = static_cast<long long>(a.units) * S_new * a.vec_per_row;
    long long blocks = (total + 255) / 256;
    const long long cap_blocks = static_cast<long long>(di->sms) * 8;
    if (blocks > cap_blocks) blocks = cap_blocks;
    return launch_pdl(kv_append_kernel, dim3(static_cast<unsigned>(blocks), 2), dim3(256), 0, stream, a) == cudaSuccess
               ? E2D2_OK
               : E2D2_ERR_CUDA;
}
}  // namespace

e2d2_status e2d2_kv_cache_append(void* k_cache, void* v_cache, int capacity, int P, const void* k_new,
                                 const void* v_new, int S_new, e2d2_dims dims, cudaStream_t stream) {
    return append_call(k_cache, v_cache, capacity, P, nullptr, k_new, v_new, S_new, dims, stream);
}

e2d2_status e2d2_kv_cache_append_ragged(void* k_cache, void* v_cache, int capacity, const int* P_dev,
                                        const void* k_new, const void* v_new, int S_new, e2d2_dims dims,
                                        cudaStream_t stream) {
    if (!P_dev) return E2D2_ERR_INVALID_ARG;
    return append_call(k_cache, v_cache, capacity, 0, P_dev, k_new, v_new, S_new, dims, stream);
}

e2d2_status e2d2_last_device_error(cudaStream_t stream) {
    DeviceInfo* di = nullptr;
    e2d2_status s = device_info(&di);
    if (s != E2D2_OK) return s;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return E2D2_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return E2D2_ERR_CUDA;
    if (word != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return E2D2_ERR_CUDA;
        return (word & kErrDeviceCheck) ? E2D2_ERR_DEVICE_CHECK : E2D2_ERR_TIMEOUT;
    }
    return E2D2_OK;
}

e2d2_status e2d2_debug_set_wait_test(unsigned long long wait_limit_ns, unsigned long long producer_delay_ns) {
    DeviceInfo* di = nullptr;
    const e2d2_status s = device_info(&di);
    if (s != E2D2_OK) return s;
    const unsigned long long limit = wait_limit_ns ? wait_limit_ns : kWaitTimeoutNs;
    if (cudaMemcpyToSymbol(g_wait_limit_ns, &limit, sizeof(limit)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_test_producer_delay_ns, &producer_delay_ns, sizeof(producer_delay_ns)) != cudaSuccess)
        return E2D2_ERR_CUDA;
    return E2D2_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// Sampling step without any allocation: for callers that cannot allocate device memory.
//
// Some callers have no way to obtain a workspace: a serving engine that hands (nearly) all of
// HBM to its own KV-cache pool at start-up and offers plugins no allocator, or a caller whose
// hot path may not call cudaMalloc because that call can synchronise the device.  This entry
// point takes the split-KV scratch from a file-scope device array instead.  The array
// (kNoAllocScratchBytes) is reserved on every GPU that loads this library until the process
// exits.  Every call shares it and it keeps the last call's contents: the per-CTA ticket words
// are cleared (cudaMemsetAsync, which allocates nothing) before each launch, and the partial
// slots are always written before they are read.  Calls that overlap on the GPU (different
// streams, or different host threads on the same device) race on the array.
// ---------------------------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = E2D2_SAMPLE_NOALLOC_MAX_BYTES;  // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
struct NoAllocScratch {
    bool ready = false;
    void* ptr = nullptr;  // device address of g_noalloc_scratch on this device
};
std::mutex g_noalloc_mutex;
NoAllocScratch g_noalloc[kMaxDevices];

// The host-side name of g_noalloc_scratch is only a stand-in; the device address comes from
// cudaGetSymbolAddress, once per device, with that device current.
e2d2_status noalloc_scratch(void** ptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return E2D2_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    NoAllocScratch& s = g_noalloc[dev];
    if (!s.ready) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return E2D2_ERR_CUDA;
        s.ptr = p;
        s.ready = true;
    }
    *ptr = s.ptr;
    return E2D2_OK;
}
}  // namespace

extern "C" {

e2d2_status e2d2_attn_decoder_sample_noalloc(const void* q_blk, const void* k_cache, const void* v_cache,
                                             int capacity, int P, const void* k_blk, const void* v_blk,
                                             void* out, float* lse, e2d2_dims dims, int S,
                                             cudaStream_t stream) {
    if (!q_blk || !k_cache || !v_cache || !k_blk || !v_blk || !out) return E2D2_ERR_INVALID_ARG;
    const e2d2_status sd = check_dims(dims);
    if (sd != E2D2_OK) return sd;
    if (S <= 0 || capacity < 0 || P < 0) return E2D2_ERR_INVALID_ARG;
    const size_t need = e2d2_attn_decoder_sample_workspace(dims, S, capacity);
    if (need == 0) return E2D2_ERR_INVALID_ARG;
    if (need > kNoAllocScratchBytes) return E2D2_ERR_WORKSPACE;  // shape needs more than the array
    void* scratch = nullptr;
    e2d2_status s = noalloc_scratch(&scratch);
    if (s != E2D2_OK) return s;
    // Every check first: an error return must leave nothing queued on the stream.
    SampleLaunch sl;
    s = sample_prepare(false, q_blk, k_cache, v_cache, capacity, P, nullptr, k_blk, v_blk, out, lse, dims, S, scratch,
                       kNoAllocScratchBytes, &sl);
    if (s != E2D2_OK) return s;
    // Ticket words must start at zero; they occupy the first kSampleMaxCtas ints.
    if (cudaMemsetAsync(scratch, 0, kSampleMaxCtas * sizeof(int), stream) != cudaSuccess) return E2D2_ERR_CUDA;
    return sample_launch(sl, stream);
}

}  // extern "C"
