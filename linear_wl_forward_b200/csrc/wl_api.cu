// C ABI of the theta-bundle linear: argument checks, the per-device scratch
// pool, tensor-map encoding and kernel selection.  Declarations and the
// contract of every entry point are in include/wl.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <memory>
#include <mutex>
#include <unordered_map>

#include "../../include/wl.h"
#include "wl_internal.h"

namespace wl {

namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up through the runtime so that the
// library needs no libcuda at link time.
EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}
}  // namespace

wl_status encode_map_2d(CUtensorMap *m, const void *ptr, uint64_t cols, uint64_t rows, uint64_t ld,
                        uint32_t box_cols, uint32_t box_rows, bool swizzle128) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return WL_ERR_CUDA;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {ld * 2};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides,
                          box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? WL_OK : WL_ERR_CUDA;
}

wl_status encode_map_2d_u32(CUtensorMap *m, const void *ptr, uint64_t cols, uint64_t rows, uint64_t ld_bytes,
                            uint32_t box_cols, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return WL_ERR_CUDA;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {ld_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? WL_OK : WL_ERR_CUDA;
}

wl_status encode_map_1d_f32(CUtensorMap *m, const void *ptr, uint64_t n, uint32_t box) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return WL_ERR_CUDA;
    const cuuint64_t dims[1] = {n};
    const cuuint64_t strides[1] = {n * 4};  // not read for a rank-1 map
    const cuuint32_t bx[1] = {box};
    const cuuint32_t estr[1] = {1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 1, const_cast<void *>(ptr), dims, strides, bx, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? WL_OK : WL_ERR_CUDA;
}

wl_status encode_map_3d(CUtensorMap *m, const void *ptr, uint64_t d0, uint64_t d1, uint64_t d2,
                        uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1,
                        uint32_t b2, bool bytes_unswizzled) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return WL_ERR_CUDA;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
    const cuuint32_t box[3] = {b0, b1, b2};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, bytes_unswizzled ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                          const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          bytes_unswizzled ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? WL_OK : WL_ERR_CUDA;
}

namespace {

// GEMM operand maps: box_rows x 64 elements.
wl_status make_map(CUtensorMap *m, const void *ptr, uint64_t cols, uint64_t rows, uint64_t ld,
                   uint32_t box_rows) {
    return encode_map_2d(m, ptr, cols, rows, ld, 64, box_rows);
}

constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per device-side wait
constexpr int kMaxDevices = 64;
std::atomic<unsigned long long> g_wait_limit_ns{kWaitLimitNs};

enum Slot {
    kSlotT = 0,
    kSlotTPart,
    kSlotVt,
    kSlotPart,
    kSlotTileCnt,  // zeroed when allocated; the kernels leave it zero
    kSlotUPad0,
    kSlotXh = kSlotUPad0 + kMaxSeg,  // NVFP4: permuted x in f16
    kSlotFp4Part,                    // NVFP4: slice partial sums of V^T x
    kSlotFp4T,                       // NVFP4: V^T x
    kSlotFp4Cnt,                     // NVFP4: prep group / projection counters (zeroed; self-resetting)
    kSlotFp4G,                       // NVFP4: group sums of V^T x
    kSlotFp4Blk,                     // NVFP4 ring: partial sums of blocks split between CTAs
    kSlotFp4BCnt,                    // NVFP4 ring: CTAs done per split block (zeroed; self-resetting)
    kNumSlots
};

struct DevicePool {
    bool ready = false;
    int num_sms = 0;
    int major = 0;
    int *words = nullptr;  // [0] status, [1] probe flag (never set), [8..15] counters
    void *buf[kNumSlots] = {};
    size_t cap[kNumSlots] = {};
};

std::mutex g_mu;
DevicePool g_pool[kMaxDevices];

wl_status from_cuda(cudaError_t e) { return e == cudaSuccess ? WL_OK : WL_ERR_CUDA; }

wl_status pool_for_current_device(DevicePool **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return WL_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return WL_ERR_UNSUPPORTED;
    DevicePool &p = g_pool[dev];
    if (!p.ready) {
        if (cudaDeviceGetAttribute(&p.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&p.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
            return WL_ERR_CUDA;
        if (cudaMalloc(&p.words, 64 * sizeof(int)) != cudaSuccess) return WL_ERR_NOMEM;
        if (cudaMemset(p.words, 0, 64 * sizeof(int)) != cudaSuccess) return WL_ERR_CUDA;
        if (cudaDeviceSynchronize() != cudaSuccess) return WL_ERR_CUDA;
        p.ready = true;
    }
    if (p.major != 10) return WL_ERR_UNSUPPORTED;  // kernels are built for sm_100a only
    *out = &p;
    return WL_OK;
}

// Grow-only scratch.  Growing waits for the device so no kernel still uses
// the old buffer; steady-state calls of one shape never reach cudaMalloc.
wl_status scratch(DevicePool &p, int slot, size_t bytes, void **out, bool zeroed = false) {
    if (bytes == 0) bytes = 16;
    if (p.cap[slot] < bytes) {
        size_t want = std::max(bytes, p.cap[slot] * 2);
        want = (want + (2u << 20) - 1) & ~size_t((2u << 20) - 1);
        if (p.buf[slot]) {
            if (cudaDeviceSynchronize() != cudaSuccess) return WL_ERR_CUDA;
            cudaFree(p.buf[slot]);
            p.buf[slot] = nullptr;
            p.cap[slot] = 0;
        }
        if (cudaMalloc(&p.buf[slot], want) != cudaSuccess) {
            cudaGetLastError();
            return WL_ERR_NOMEM;
        }
        if (zeroed && cudaMemset(p.buf[slot], 0, want) != cudaSuccess) return WL_ERR_CUDA;
        p.cap[slot] = want;
    }
    *out = p.buf[slot];
    return WL_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------- validation --
// Pure host checks; touches no CUDA API, so it is testable without a GPU.
wl_status validate(const wl_bf16 *x, int M, int K, const wl_proj *projs, int P, wl_path path) {
    if (!projs) return WL_ERR_INVALID_ARG;
    if (P < 1 || P > WL_MAX_PROJ) return P < 1 ? WL_ERR_INVALID_ARG : WL_ERR_UNSUPPORTED;
    if (M < 0 || K < 0) return WL_ERR_INVALID_ARG;
    if (path != WL_PATH_AUTO && path != WL_PATH_DECODE && path != WL_PATH_GEMM && path != WL_PATH_ROWS &&
        path != WL_PATH_RING)
        return WL_ERR_INVALID_ARG;
    for (int i = 0; i < P; ++i) {
        const wl_proj &q = projs[i];
        if (q.N < 0 || q.r < 0) return WL_ERR_INVALID_ARG;
        if (q.r > WL_MAX_RANK) return WL_ERR_UNSUPPORTED;
        if (M > 0 && q.N > 0) {
            if (!q.y || !q.s || (K > 0 && !q.W0)) return WL_ERR_INVALID_ARG;
            if (q.r > 0 && K > 0 && (!q.U || !q.V)) return WL_ERR_INVALID_ARG;
        }
    }
    if (M > 0 && K > 0 && !x) return WL_ERR_INVALID_ARG;
    if (K % 8 != 0) return WL_ERR_ALIGNMENT;
    if (M > 0 && K > 0) {
        if (!aligned16(x)) return WL_ERR_ALIGNMENT;
        for (int i = 0; i < P; ++i)
            if (projs[i].N > 0 && !aligned16(projs[i].W0)) return WL_ERR_ALIGNMENT;
    }
    if ((path == WL_PATH_DECODE || path == WL_PATH_ROWS) && M > WL_DECODE_MAX_M) return WL_ERR_UNSUPPORTED;
    return WL_OK;
}

int round_up(int v, int m) { return (v + m - 1) / m * m; }

// The prefetch ranges of a call, each trimmed to its 16-byte-aligned interior
// (empty ones dropped).  Pure host code.
wl_status build_prefetch(const wl_range *ranges, int n, PrefetchList &pf) {
    std::memset(&pf, 0, sizeof pf);
    if (n < 0 || n > WL_MAX_PREFETCH || (n > 0 && !ranges)) return WL_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        if (ranges[i].bytes == 0) continue;
        if (!ranges[i].ptr) return WL_ERR_INVALID_ARG;
        const uintptr_t a = reinterpret_cast<uintptr_t>(ranges[i].ptr);
        const uintptr_t lo = (a + 15) & ~uintptr_t(15);
        const uintptr_t hi = (a + ranges[i].bytes) & ~uintptr_t(15);
        if (hi <= lo) continue;
        pf.ptr[pf.n] = reinterpret_cast<const uint8_t *>(lo);
        pf.bytes[pf.n] = hi - lo;
        pf.total += hi - lo;
        ++pf.n;
    }
    return WL_OK;
}

// WL_PATH_AUTO: the weight-streaming decode kernel for up to 4 tokens, and
// for up to WL_DECODE_MAX_M tokens when the call is narrow (its projections
// total fewer than 8192 output rows).  Wider calls with 5..16 tokens go to the
// tensor-core GEMM, which keeps x out of shared memory and fills every SM with
// tiles; measured on B200 (one call at a time, rotating buffers > L2):
//   stacked gate/up 2 x 21504 x 5376, M = 8 / 16: GEMM 162 / 152 us, decode 252 / 242 us
//   stacked gate/up 2 x 4096 x 1152, M = 8: GEMM 26.9 us, decode 30.1 us
//   down 5376 x 21504, M = 8 / 16: decode 107 / 141 us, GEMM 231 / 234 us
//   q/k/v 1536 x 1152, M = 8: decode 19.5 us, GEMM 22.9 us
// Large calls of at most 8 tokens take the persistent ring: at least 64 MB
// of bf16 weights (the Gemma-4-31B projections; measured against the other
// kernels, us at M = 1 / 8: gate/up 88.7 / 126.6 against 122.5 (decode) /
// 133.7 (GEMM), down 50.8 / 76.7 against 72.0 / 106.2, q/k/v 45.9 against
// 66.3 at M = 1).
bool auto_ring(int M, int K, const wl_proj *projs, int P) {
    if (M > kFp4MaxM) return false;
    long long rows = 0;
    for (int i = 0; i < P; ++i) rows += projs[i].N;
    return 2LL * rows * K >= (64LL << 20);
}

bool auto_decode(int M, const wl_proj *projs, int P) {
    if (M > WL_DECODE_MAX_M) return false;
    if (M <= 4) return true;
    long long rows = 0;
    for (int i = 0; i < P; ++i) rows += projs[i].N;
    return rows < 8192;
}

// ------------------------------------------------------------------ paths --
// Fills the decode parameters of a call; false if no projection has rows.
bool build_decode_params(const wl_bf16 *x, int M, int K, const wl_proj *projs, int P,
                         DecodeParams &dp) {
    std::memset(&dp, 0, sizeof dp);
    int total = 0, t_off = 0, nseg = 0;
    for (int i = 0; i < P; ++i) {
        const wl_proj &q = projs[i];
        if (q.N == 0) continue;
        DecodeSeg &sg = dp.a.seg[nseg++];
        sg.W0 = reinterpret_cast<const __nv_bfloat16 *>(q.W0);
        sg.s = q.s;
        sg.U = reinterpret_cast<const __nv_bfloat16 *>(q.U);
        sg.V = reinterpret_cast<const __nv_bfloat16 *>(q.V);
        sg.y = reinterpret_cast<__nv_bfloat16 *>(q.y);
        sg.N = q.N;
        sg.r = q.r;
        sg.t_off = t_off;
        total += q.N;
        t_off += q.r;
    }
    if (total == 0) return false;
    dp.a.nseg = nseg;
    dp.a.M = M;
    dp.a.K = K;
    dp.a.t_ld = t_off;
    dp.a.x = reinterpret_cast<const __nv_bfloat16 *>(x);
    return true;
}

// Returns WL_ERR_UNSUPPORTED if the shape cannot take the decode kernel.
// Decode plans of recent calls, keyed by everything the plan depends on (the
// call's pointers and sizes).  A decode step issues the same calls with the
// same buffers every time, so a hit skips the tensor-map encoding and the
// planning; only the scratch pointers are filled in per call.
struct DecodeKey {
    const void *x;
    int M, K, P;
    wl_proj projs[kMaxSeg];
    bool operator==(const DecodeKey &o) const { return std::memcmp(this, &o, sizeof *this) == 0; }
};

struct DecodeKeyHash {
    size_t operator()(const DecodeKey &k) const {
        // FNV-1a over the key's bytes
        const unsigned char *b = reinterpret_cast<const unsigned char *>(&k);
        uint64_t h = 1469598103934665603ull;
        for (size_t i = 0; i < sizeof k; ++i) h = (h ^ b[i]) * 1099511628211ull;
        return (size_t)h;
    }
};

struct DecodeEntry {
    DecodeParams dp;
    DecodePlan plan;
    wl_status status;  // WL_OK or WL_ERR_UNSUPPORTED (the shape cannot take the decode kernel)
};

constexpr size_t kDecodeCacheMax = 4096;
std::unordered_map<DecodeKey, std::unique_ptr<DecodeEntry>, DecodeKeyHash> g_decode_cache[kMaxDevices];

wl_status run_decode(DevicePool &pool, const wl_bf16 *x, int M, int K, const wl_proj *projs, int P,
                     const PrefetchList &pf, cudaStream_t stream) {
    DecodeKey key;
    std::memset(&key, 0, sizeof key);  // padding bytes take part in the comparison
    key.x = x;
    key.M = M;
    key.K = K;
    key.P = P;
    std::memcpy(key.projs, projs, sizeof(wl_proj) * P);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return WL_ERR_CUDA;
    auto &cache = g_decode_cache[dev];
    auto it = cache.find(key);
    if (it == cache.end()) {
        if (cache.size() >= kDecodeCacheMax) cache.clear();
        auto e = std::make_unique<DecodeEntry>();
        if (!build_decode_params(x, M, K, projs, P, e->dp)) return WL_OK;
        e->status = plan_decode(e->dp, pool.num_sms, &e->plan);
        if (e->status != WL_OK && e->status != WL_ERR_UNSUPPORTED) return e->status;
        it = cache.emplace(key, std::move(e)).first;
    }
    DecodeEntry &e = *it->second;
    if (e.status != WL_OK) return e.status;
    DecodeParams &dp = e.dp;
    const DecodePlan &plan = e.plan;
    dp.a.status = pool.words;
    dp.a.sync = reinterpret_cast<unsigned int *>(pool.words + 8);
    dp.a.timeout_ns = wait_limit_ns();
    dp.pf = pf;
    if (plan.tpart_bytes) {
        void *tp = nullptr;
        wl_status st = scratch(pool, kSlotTPart, plan.tpart_bytes, &tp);
        if (st != WL_OK) return st;
        dp.a.Tpart = static_cast<float *>(tp);
    }
    return from_cuda(launch_decode(dp, plan, stream));
}

// Row-stream plans of recent calls, keyed like the decode plans (no tensor
// maps: planning is cheap, but a decode step repeats its calls).
struct RowsEntry {
    RowsParams rp;
    wl_status status;  // WL_OK or WL_ERR_UNSUPPORTED (the call does not fit the kernel)
};
std::unordered_map<DecodeKey, std::unique_ptr<RowsEntry>, DecodeKeyHash> g_rows_cache[kMaxDevices];

// Returns WL_ERR_UNSUPPORTED (launching nothing) if the call does not fit the
// row-stream kernel.
wl_status run_rows(DevicePool &pool, const wl_bf16 *x, int M, int K, const wl_proj *projs, int P,
                   const PrefetchList &pf, cudaStream_t stream) {
    DecodeKey key;
    std::memset(&key, 0, sizeof key);
    key.x = x;
    key.M = M;
    key.K = K;
    key.P = P;
    std::memcpy(key.projs, projs, sizeof(wl_proj) * P);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return WL_ERR_CUDA;
    auto &cache = g_rows_cache[dev];
    auto it = cache.find(key);
    if (it == cache.end()) {
        if (cache.size() >= kDecodeCacheMax) cache.clear();
        auto e = std::make_unique<RowsEntry>();
        e->status = plan_rows(e->rp, M, K, projs, P, pool.num_sms);
        if (e->status != WL_OK && e->status != WL_ERR_UNSUPPORTED) return e->status;
        it = cache.emplace(key, std::move(e)).first;
    }
    RowsEntry &e = *it->second;
    if (e.status != WL_OK) return e.status;
    e.rp.x = reinterpret_cast<const __nv_bfloat16 *>(x);
    e.rp.status = pool.words;
    e.rp.timeout_ns = wait_limit_ns();
    e.rp.pf = pf;
    return from_cuda(launch_rows(e.rp, stream));
}

wl_status run_gemm(DevicePool &pool, const wl_bf16 *x, int M, int K, const wl_proj *projs, int P,
                   const PrefetchList &pf, cudaStream_t stream) {
    // Column layout of T: each projection with r > 0 gets round_up(r, 64) columns.
    int t_cols = 0;
    int t_col[kMaxSeg] = {};
    for (int i = 0; i < P; ++i) {
        t_col[i] = t_cols;
        if (projs[i].N > 0 && projs[i].r > 0) t_cols += round_up(projs[i].r, 64);
    }
    __nv_bfloat16 *T = nullptr;
    wl_status st;
    if (t_cols > 0) {
        void *vt = nullptr, *t = nullptr;
        if ((st = scratch(pool, kSlotVt, (size_t)t_cols * K * 2, &vt)) != WL_OK) return st;
        if ((st = scratch(pool, kSlotT, (size_t)M * t_cols * 2, &t)) != WL_OK) return st;
        __nv_bfloat16 *Vt = static_cast<__nv_bfloat16 *>(vt);
        T = static_cast<__nv_bfloat16 *>(t);
        TransposeVArgs ta;
        std::memset(&ta, 0, sizeof ta);
        ta.K = K;
        ta.Vt = Vt;
        for (int i = 0; i < P; ++i) {
            const wl_proj &q = projs[i];
            if (q.N == 0 || q.r == 0) continue;
            ta.V[ta.n] = reinterpret_cast<const __nv_bfloat16 *>(q.V);
            ta.r[ta.n] = q.r;
            ta.r_pad[ta.n] = round_up(q.r, 64);
            ta.row[ta.n] = t_col[i];
            ++ta.n;
        }
        if (launch_transpose_v(ta, stream) != cudaSuccess) return WL_ERR_CUDA;
        // T = x V for all projections at once (plain GEMM against the stacked V^T).
        GemmParams tp;
        std::memset(&tp, 0, sizeof tp);
        const int bn = t_cols >= 256 ? 256 : t_cols;
        if ((st = make_map(&tp.tm_a, x, K, M, K, kGemmBM)) != WL_OK) return st;
        tp.tm_t = tp.tm_a;
        if ((st = make_map(&tp.tm_b[0], Vt, K, t_cols, K, bn)) != WL_OK) return st;
        tp.tm_u[0] = tp.tm_b[0];
        tp.nseg = 1;
        tp.M = M;
        tp.K = K;
        tp.BN = bn;
        tp.num_m_tiles = (M + kGemmBM - 1) / kGemmBM;
        tp.seg[0].s = nullptr;
        tp.seg[0].y = T;
        tp.seg[0].N = t_cols;
        tp.seg[0].ldy = t_cols;
        tp.seg[0].lr_blocks = 0;
        tp.seg[0].tile_begin = 0;
        tp.num_tiles = tp.num_m_tiles * ((t_cols + bn - 1) / bn);
        tp.ksplit = 1;
        tp.kb_split = (K + kGemmBK - 1) / kGemmBK;
        set_gemm_stages(tp);
        tp.status = pool.words;
        tp.timeout_ns = wait_limit_ns();
        if (launch_gemm(tp, pool.num_sms, stream) != cudaSuccess) return WL_ERR_CUDA;
    }

    GemmParams gp;
    std::memset(&gp, 0, sizeof gp);
    const int nkb = (K + kGemmBK - 1) / kGemmBK;
    const bool swap = M <= kGemmSwapMaxM;
    int bn = kGemmMaxBN;
    if (swap) {
        // Few tokens: swap the operands so the 128-row MMA side runs over the
        // output rows (W0 / U tiles) and the tokens are the MMA's N (mp).
        bn = kGemmBM;
        gp.swap = 1;
        gp.mp = round_up(M, 16);
    } else {
        // Tile width: the widest of 256, 128, 64 that still gives every SM a
        // tile.  Narrower than 64 would make the x tile, re-read per tile,
        // outweigh W0.
        const int m_tiles = (M + kGemmBM - 1) / kGemmBM;
        while (bn > 64) {
            int n_tiles = 0;
            for (int i = 0; i < P; ++i) n_tiles += (projs[i].N + bn - 1) / bn;
            if (m_tiles * n_tiles >= pool.num_sms) break;
            bn /= 2;
        }
    }
    const uint32_t xb_rows = swap ? (uint32_t)gp.mp : (uint32_t)kGemmBM;
    if ((st = make_map(&gp.tm_a, x, K, M, K, xb_rows)) != WL_OK) return st;
    if (t_cols > 0) {
        if ((st = make_map(&gp.tm_t, T, t_cols, M, t_cols, xb_rows)) != WL_OK) return st;
    } else {
        gp.tm_t = gp.tm_a;
    }
    gp.M = M;
    gp.K = K;
    gp.BN = bn;
    gp.num_m_tiles = swap ? 1 : (M + kGemmBM - 1) / kGemmBM;
    int tiles = 0, nseg = 0;
    for (int i = 0; i < P; ++i) {
        const wl_proj &q = projs[i];
        if (q.N == 0) continue;
        const int sidx = nseg++;
        if ((st = make_map(&gp.tm_b[sidx], q.W0, K, q.N, K, bn)) != WL_OK) return st;
        GemmSeg &sg = gp.seg[sidx];
        sg.s = q.s;
        sg.y = reinterpret_cast<__nv_bfloat16 *>(q.y);
        sg.N = q.N;
        sg.ldy = q.N;
        sg.t_col = t_col[i];
        sg.tile_begin = tiles;
        tiles += gp.num_m_tiles * ((q.N + bn - 1) / bn);
        if (q.r > 0) {
            const int r_pad = round_up(q.r, 64);
            sg.lr_blocks = r_pad / 64;
            if (q.r % 8 == 0 && aligned16(q.U)) {
                if ((st = make_map(&gp.tm_u[sidx], q.U, q.r, q.N, q.r, bn)) != WL_OK) return st;
            } else {
                void *up = nullptr;
                if ((st = scratch(pool, kSlotUPad0 + sidx, (size_t)q.N * r_pad * 2, &up)) != WL_OK)
                    return st;
                if (launch_pad_u(reinterpret_cast<const __nv_bfloat16 *>(q.U), q.N, q.r, r_pad,
                                 static_cast<__nv_bfloat16 *>(up), stream) != cudaSuccess)
                    return WL_ERR_CUDA;
                if ((st = make_map(&gp.tm_u[sidx], up, r_pad, q.N, r_pad, bn)) != WL_OK) return st;
            }
        } else {
            sg.lr_blocks = 0;
            gp.tm_u[sidx] = gp.tm_b[sidx];
        }
    }
    if (tiles == 0) return WL_OK;
    gp.nseg = nseg;
    gp.num_tiles = tiles;
    // K ranges per tile: in swap mode, enough to fill the SMs when the output
    // rows alone give too few tiles (each range keeps >= 8 K blocks).
    // Only when the output tiles alone leave SMs idle; the smallest split that
    // keeps 80% of the SMs busy (the ranges' sums cost a reduction).
    gp.ksplit = 1;
    if (swap && tiles < pool.num_sms) {
        for (int ks = 2; ks <= kGemmMaxKSplit; ++ks) {
            const int kbs = (nkb + ks - 1) / ks;
            if (kbs < 8) break;
            const int eff_ks = (nkb + kbs - 1) / kbs;
            const long long u = (long long)tiles * eff_ks;
            const long long waves = (u + pool.num_sms - 1) / pool.num_sms;
            gp.ksplit = eff_ks;
            if ((double)u / (double)(waves * pool.num_sms) >= 0.8) break;
        }
    }
    gp.kb_split = (nkb + gp.ksplit - 1) / gp.ksplit;
    gp.ksplit = (nkb + gp.kb_split - 1) / gp.kb_split;
    if (gp.ksplit > 1) {
        void *part = nullptr, *cnt = nullptr;
        const size_t pf = (size_t)(gp.ksplit + 1) * tiles * gp.mp * kGemmBM;
        if ((st = scratch(pool, kSlotPart, pf * sizeof(float), &part)) != WL_OK) return st;
        if ((st = scratch(pool, kSlotTileCnt, (size_t)tiles * sizeof(unsigned), &cnt, true)) != WL_OK)
            return st;
        gp.part = static_cast<float *>(part);
        gp.tile_cnt = static_cast<unsigned int *>(cnt);
    }
    set_gemm_stages(gp);
    gp.status = pool.words;
    gp.timeout_ns = wait_limit_ns();
    gp.pf = pf;
    return from_cuda(launch_gemm(gp, pool.num_sms, stream));
}

// Scratch and launch of a planned NVFP4 (or bf16-ring) call; g_mu held.
wl_status fp4_run(DevicePool &pool, Fp4Params &fp, cudaStream_t stream) {
    wl_status st;
    const int M = fp.M;
    const size_t tl = (size_t)(fp.t_ld > 0 ? fp.t_ld : 1);
    void *xq = nullptr, *tp = nullptr, *gp = nullptr, *tt = nullptr, *cnt = nullptr;
    if ((st = scratch(pool, kSlotXh, fp4_xq_halves(fp) * 2, &xq)) != WL_OK) return st;
    if ((st = scratch(pool, kSlotFp4Part, (size_t)fp.slices * M * tl * sizeof(float), &tp)) != WL_OK) return st;
    if ((st = scratch(pool, kSlotFp4G, (size_t)fp.ngrp * M * tl * sizeof(float), &gp)) != WL_OK) return st;
    if ((st = scratch(pool, kSlotFp4T, (size_t)M * tl * sizeof(float), &tt)) != WL_OK) return st;
    if ((st = scratch(pool, kSlotFp4Cnt, (size_t)(kMaxSeg * (fp.ngrp + 1)) * sizeof(unsigned), &cnt, true)) != WL_OK)
        return st;
    fp.xq = static_cast<__half *>(xq);
    fp.Tpart = static_cast<float *>(tp);
    fp.Gpart = static_cast<float *>(gp);
    fp.T = static_cast<float *>(tt);
    fp.cnt = static_cast<unsigned int *>(cnt);
    if (fp.ring) {
        void *pa = nullptr, *bc = nullptr;
        if ((st = scratch(pool, kSlotFp4Blk, (size_t)fp.grid * 2 * 16 * kFp4MaxM * sizeof(float2), &pa)) != WL_OK)
            return st;
        if ((st = scratch(pool, kSlotFp4BCnt, (size_t)fp.total_blocks * sizeof(unsigned), &bc, true)) != WL_OK)
            return st;
        fp.parts = static_cast<float2 *>(pa);
        fp.bcnt = static_cast<unsigned int *>(bc);
    }
    return from_cuda(launch_fp4(fp, stream));
}

// The bf16 forward on the persistent ring (prep launch for V^T x and the
// permuted x, then the ring): WL_ERR_UNSUPPORTED for calls it does not take.
wl_status ring_params(Fp4Params &fp, const wl_bf16 *x, int M, int K, const wl_proj *projs, int P, int num_sms,
                      bool encode_maps) {
    if (M < 1 || M > kFp4MaxM) return WL_ERR_UNSUPPORTED;
    std::memset(&fp, 0, sizeof fp);
    int blocks = 0, t_off = 0, nr = 0;
    for (int i = 0; i < P; ++i) {
        const wl_proj &q = projs[i];
        if (q.N == 0) continue;
        if (q.r % 8 != 0 || q.r > kFp4RingMaxRank) return WL_ERR_UNSUPPORTED;
        if (q.r > 0 && (!aligned16(q.U) || !aligned16(q.V))) return WL_ERR_UNSUPPORTED;
        Fp4Seg &sg = fp.seg[fp.nseg++];
        sg.codes = reinterpret_cast<const uint8_t *>(q.W0);
        sg.scales = nullptr;
        sg.ts = 1.f;
        sg.s = q.s;
        sg.U = reinterpret_cast<const __nv_bfloat16 *>(q.U);
        sg.V = reinterpret_cast<const __nv_bfloat16 *>(q.V);
        sg.y = reinterpret_cast<__nv_bfloat16 *>(q.y);
        sg.N = q.N;
        sg.r = q.r;
        sg.blk_begin = blocks;
        sg.t_off = t_off;
        blocks += (q.N + 15) / 16;
        t_off += q.r;
        nr += q.r > 0;
    }
    if (fp.nseg == 0) return WL_ERR_UNSUPPORTED;
    fp.bf16 = 1;
    fp.M = M;
    fp.K = K;
    fp.total_blocks = blocks;
    fp.t_ld = t_off;
    fp.nr = nr;
    fp.x = reinterpret_cast<const __nv_bfloat16 *>(x);
    return plan_fp4(fp, num_sms, encode_maps);
}

wl_status run_ring(DevicePool &pool, const wl_bf16 *x, int M, int K, const wl_proj *projs, int P,
                   cudaStream_t stream) {
    static Fp4Params fp;  // guarded by g_mu
    wl_status st = ring_params(fp, x, M, K, projs, P, pool.num_sms, true);
    if (st != WL_OK) return st;
    fp.status = pool.words;
    fp.timeout_ns = wait_limit_ns();
    return fp4_run(pool, fp, stream);
}

wl_status forward(const wl_bf16 *x, int M, int K, const wl_proj *projs, int P, wl_path path,
                  const wl_range *prefetch, int nprefetch, void *stream_ptr) {
    wl_status st = validate(x, M, K, projs, P, path);
    if (st != WL_OK) return st;
    PrefetchList pf;
    if ((st = build_prefetch(prefetch, nprefetch, pf)) != WL_OK) return st;
    bool any = false;
    for (int i = 0; i < P; ++i) any = any || projs[i].N > 0;
    if (M == 0 || !any) return WL_OK;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    if (K == 0) {  // W0 x = 0 and V^T x = 0: y = 0
        for (int i = 0; i < P; ++i)
            if (projs[i].N > 0 &&
                cudaMemsetAsync(projs[i].y, 0, (size_t)M * projs[i].N * 2, stream) != cudaSuccess)
                return WL_ERR_CUDA;
        return WL_OK;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    DevicePool *pool = nullptr;
    if ((st = pool_for_current_device(&pool)) != WL_OK) return st;
    if (path == WL_PATH_AUTO && auto_ring(M, K, projs, P)) {
        st = run_ring(*pool, x, M, K, projs, P, stream);
        if (st != WL_ERR_UNSUPPORTED) return st;
    }
    if (path == WL_PATH_AUTO && auto_decode(M, projs, P)) {
        // Each decode kernel declines shapes it cannot hold (before launching
        // anything): short calls take the row-stream kernel, the rest the
        // weight-streaming one, and what neither holds the tensor-core GEMM.
        st = run_rows(*pool, x, M, K, projs, P, pf, stream);
        if (st != WL_ERR_UNSUPPORTED) return st;
        st = run_decode(*pool, x, M, K, projs, P, pf, stream);
        return st == WL_ERR_UNSUPPORTED ? run_gemm(*pool, x, M, K, projs, P, pf, stream) : st;
    }
    if (path == WL_PATH_ROWS) return run_rows(*pool, x, M, K, projs, P, pf, stream);
    if (path == WL_PATH_RING) return run_ring(*pool, x, M, K, projs, P, stream);
    return path == WL_PATH_DECODE ? run_decode(*pool, x, M, K, projs, P, pf, stream)
                                  : run_gemm(*pool, x, M, K, projs, P, pf, stream);
}

}  // namespace

unsigned long long wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

}  // namespace wl

extern "C" {

wl_status wl_set_wait_limit(long long limit_ns) {
    if (limit_ns < 0 || limit_ns > 10000000000LL) return WL_ERR_INVALID_ARG;
    wl::g_wait_limit_ns.store(limit_ns == 0 ? wl::kWaitLimitNs : (unsigned long long)limit_ns,
                              std::memory_order_relaxed);
    return WL_OK;
}

wl_status wl_linear_forward(const wl_bf16 *x, const wl_bf16 *W0, const float *s, const wl_bf16 *U,
                            const wl_bf16 *V, wl_bf16 *y, int M, int N, int K, int r, void *stream) {
    wl_proj p;
    p.W0 = W0;
    p.s = s;
    p.U = U;
    p.V = V;
    p.y = y;
    p.N = N;
    p.r = r;
    return wl::forward(x, M, K, &p, 1, WL_PATH_AUTO, nullptr, 0, stream);
}

wl_status wl_stacked_forward(const wl_bf16 *x, int M, int K, const wl_proj *projs, int P,
                             void *stream) {
    return wl::forward(x, M, K, projs, P, WL_PATH_AUTO, nullptr, 0, stream);
}

wl_status wl_forward_ex(const wl_bf16 *x, int M, int K, const wl_proj *projs, int P, wl_path path,
                        void *stream) {
    return wl::forward(x, M, K, projs, P, path, nullptr, 0, stream);
}

wl_status wl_stacked_forward_prefetch(const wl_bf16 *x, int M, int K, const wl_proj *projs, int P,
                                      wl_path path, const wl_range *prefetch, int n, void *stream) {
    return wl::forward(x, M, K, projs, P, path, prefetch, n, stream);
}

const char *wl_status_string(wl_status s) {
    switch (s) {
        case WL_OK: return "ok";
        case WL_ERR_INVALID_ARG: return "invalid argument";
        case WL_ERR_ALIGNMENT: return "misaligned argument (K % 8 != 0 or pointer not 16-byte aligned)";
        case WL_ERR_UNSUPPORTED: return "unsupported (rank, projection count, path or device)";
        case WL_ERR_CUDA: return "CUDA error";
        case WL_ERR_TIMEOUT: return "device-side wait timed out";
        case WL_ERR_NOMEM: return "out of memory";
        case WL_ERR_NOT_CONVERGED: return "host SVD did not converge within its sweep limit";
    }
    return "unknown status";
}

wl_status wl_materialize_weight(const wl_bf16 *W0, const float *s, const wl_bf16 *U, const wl_bf16 *V,
                                wl_bf16 *W_eff, int N, int K, int r, void *stream) {
    if (N < 0 || K < 0 || r < 0) return WL_ERR_INVALID_ARG;
    if (r > WL_MAX_RANK) return WL_ERR_UNSUPPORTED;
    if (N == 0 || K == 0) return WL_OK;
    if (!W0 || !s || !W_eff || (r > 0 && (!U || !V))) return WL_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(wl::g_mu);
    wl::DevicePool *pool = nullptr;
    wl_status st = wl::pool_for_current_device(&pool);
    if (st != WL_OK) return st;
    return wl::from_cuda(wl::launch_materialize(
        reinterpret_cast<const __nv_bfloat16 *>(W0), s, reinterpret_cast<const __nv_bfloat16 *>(U),
        reinterpret_cast<const __nv_bfloat16 *>(V), reinterpret_cast<__nv_bfloat16 *>(W_eff), N, K, r,
        static_cast<cudaStream_t>(stream)));
}

wl_status wl_describe_decode_plan(int M, int K, const wl_proj *projs, int P, int num_sms,
                                  wl_decode_plan *out) {
    if (!out || num_sms < 1) return WL_ERR_INVALID_ARG;
    std::memset(out, 0, sizeof *out);
    // x is not part of a plan: validate the projections against an aligned stand-in
    alignas(16) static const unsigned char no_x[16] = {};
    wl_status st = wl::validate(reinterpret_cast<const wl_bf16 *>(no_x), M, K, projs, P, WL_PATH_DECODE);
    if (st != WL_OK) return st;
    out->auto_decode = wl::auto_decode(M, projs, P) ? 1 : 0;
    if (M < 1 || K < 8) return WL_ERR_UNSUPPORTED;
    static wl::DecodeParams dp;  // large (tensor maps); guarded by g_mu
    std::lock_guard<std::mutex> lock(wl::g_mu);
    if (!wl::build_decode_params(nullptr, M, K, projs, P, dp)) return WL_ERR_UNSUPPORTED;
    wl::DecodePlan plan;
    if ((st = wl::plan_decode(dp, num_sms, &plan, false)) != WL_OK) return st;
    const wl::DecodeArgs &a = dp.a;
    out->grid = plan.grid;
    out->compact = plan.small;
    out->smem_bytes = (long long)plan.smem;
    out->t_mode = a.t_mode;
    out->t_fused = a.t_fused;
    out->seg_split = a.seg_split;
    out->slots = a.slots;
    out->slot_chunks = a.slot_chunks;
    out->x_smem = a.x_smem;
    out->v_stage = a.v_stage;
    out->v_in_ring = a.v_in_ring;
    out->u_stage = a.u_stage;
    out->lag = a.lag;
    return WL_OK;
}

namespace {

// Argument checks of the NVFP4 forward; WL_OK with *trivial set when there is
// nothing to launch (M == 0, no rows, or K == 0).
wl_status nvfp4_validate(const wl_bf16 *x, int M, int K, const wl_proj_nvfp4 *projs, int P, bool *trivial) {
    using namespace wl;
    *trivial = false;
    if (!projs) return WL_ERR_INVALID_ARG;
    if (P < 1 || P > WL_MAX_PROJ) return P < 1 ? WL_ERR_INVALID_ARG : WL_ERR_UNSUPPORTED;
    if (M < 0 || K < 0) return WL_ERR_INVALID_ARG;
    bool any = false;
    for (int i = 0; i < P; ++i) {
        const wl_proj_nvfp4 &q = projs[i];
        if (q.N < 0 || q.r < 0) return WL_ERR_INVALID_ARG;
        if (q.r > WL_MAX_RANK) return WL_ERR_UNSUPPORTED;
        if (q.N == 0) continue;
        any = true;
        if (M > 0 && (!q.y || !q.s || (K > 0 && (!q.codes || !q.scales)))) return WL_ERR_INVALID_ARG;
        if (M > 0 && K > 0 && q.r > 0 && (!q.U || !q.V)) return WL_ERR_INVALID_ARG;
        if (!(q.tensor_scale > 0.f) || !(q.tensor_scale < 3.0e38f)) return WL_ERR_INVALID_ARG;
    }
    if (M > 0 && K > 0 && !x) return WL_ERR_INVALID_ARG;
    if (K % kFp4KGroup != 0) return WL_ERR_ALIGNMENT;
    if (M > 0 && K > 0) {
        if (!aligned16(x)) return WL_ERR_ALIGNMENT;
        for (int i = 0; i < P; ++i) {
            const wl_proj_nvfp4 &q = projs[i];
            if (q.N == 0) continue;
            if (!aligned16(q.codes) || (reinterpret_cast<uintptr_t>(q.scales) & 1u)) return WL_ERR_ALIGNMENT;
            if (q.r > 0 && (q.r % 8 != 0 || !aligned16(q.U) || !aligned16(q.V))) return WL_ERR_ALIGNMENT;
        }
    }
    if (M > WL_NVFP4_MAX_M) return WL_ERR_UNSUPPORTED;
    *trivial = M == 0 || !any || K == 0;
    return WL_OK;
}

// The projections with rows, in order, as kernel segments.
void nvfp4_fill(wl::Fp4Params &fp, const wl_bf16 *x, int M, int K, const wl_proj_nvfp4 *projs, int P) {
    using namespace wl;
    std::memset(&fp, 0, sizeof fp);
    int blocks = 0, t_off = 0, nr = 0;
    for (int i = 0; i < P; ++i) {
        const wl_proj_nvfp4 &q = projs[i];
        if (q.N == 0) continue;
        Fp4Seg &sg = fp.seg[fp.nseg++];
        sg.codes = q.codes;
        sg.scales = q.scales;
        sg.ts = q.tensor_scale;
        sg.s = q.s;
        sg.U = reinterpret_cast<const __nv_bfloat16 *>(q.U);
        sg.V = reinterpret_cast<const __nv_bfloat16 *>(q.V);
        sg.y = reinterpret_cast<__nv_bfloat16 *>(q.y);
        sg.N = q.N;
        sg.r = q.r;
        sg.blk_begin = blocks;
        sg.t_off = t_off;
        blocks += (q.N + 15) / 16;
        t_off += q.r;
        nr += q.r > 0;
    }
    fp.M = M;
    fp.K = K;
    fp.total_blocks = blocks;
    fp.t_ld = t_off;
    fp.nr = nr;
    fp.x = reinterpret_cast<const __nv_bfloat16 *>(x);
}

}  // namespace

wl_status wl_stacked_forward_nvfp4(const wl_bf16 *x, int M, int K, const wl_proj_nvfp4 *projs, int P,
                                   void *stream_ptr) {
    using namespace wl;
    bool trivial = false;
    wl_status st = nvfp4_validate(x, M, K, projs, P, &trivial);
    if (st != WL_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    if (trivial) {
        if (M > 0 && K == 0)
            for (int i = 0; i < P; ++i)
                if (projs[i].N > 0 &&
                    cudaMemsetAsync(projs[i].y, 0, (size_t)M * projs[i].N * 2, stream) != cudaSuccess)
                    return WL_ERR_CUDA;
        return WL_OK;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    DevicePool *pool = nullptr;
    if ((st = pool_for_current_device(&pool)) != WL_OK) return st;
    static Fp4Params fp;  // guarded by g_mu
    nvfp4_fill(fp, x, M, K, projs, P);
    fp.status = pool->words;
    fp.timeout_ns = wait_limit_ns();
    if ((st = plan_fp4(fp, pool->num_sms)) != WL_OK) return st;
    return fp4_run(*pool, fp, stream);
}

wl_status wl_describe_nvfp4_plan(int M, int K, const wl_proj_nvfp4 *projs, int P, int num_sms,
                                 wl_nvfp4_plan *out) {
    using namespace wl;
    if (!out || num_sms < 1) return WL_ERR_INVALID_ARG;
    std::memset(out, 0, sizeof *out);
    alignas(16) static const unsigned char no_x[16] = {};
    bool trivial = false;
    wl_status st = nvfp4_validate(reinterpret_cast<const wl_bf16 *>(no_x), M, K, projs, P, &trivial);
    if (st != WL_OK) return st;
    if (trivial) return WL_OK;
    static Fp4Params fp;  // guarded by g_mu
    std::lock_guard<std::mutex> lock(g_mu);
    nvfp4_fill(fp, reinterpret_cast<const wl_bf16 *>(no_x), M, K, projs, P);
    if ((st = plan_fp4(fp, num_sms, false)) != WL_OK) return st;
    out->ring = fp.ring;
    out->grid = fp.ring ? fp.grid : fp.total_blocks;
    out->stages = fp.ring ? fp.ns : 0;
    out->slot_bytes = fp.ring ? fp.slot_bytes : 0;
    out->smem_bytes = fp.ring ? fp.smem : 0;
    out->units = fp.ring ? fp.utot : 0;
    out->prep_slices = fp.slices;
    out->prep_rows = fp.kr;
    out->prep_grid = fp.slices * (fp.nr > 0 ? fp.nr : 1);
    return WL_OK;
}

wl_status wl_describe_rows_plan(int M, int K, const wl_proj *projs, int P, int num_sms, wl_rows_plan *out) {
    if (!out || num_sms < 1) return WL_ERR_INVALID_ARG;
    std::memset(out, 0, sizeof *out);
    alignas(16) static const unsigned char no_x[16] = {};
    wl_status st = wl::validate(reinterpret_cast<const wl_bf16 *>(no_x), M, K, projs, P, WL_PATH_ROWS);
    if (st != WL_OK) return st;
    static wl::RowsParams rp;  // large (tensor maps); guarded by g_mu
    std::lock_guard<std::mutex> lock(wl::g_mu);
    if ((st = wl::plan_rows(rp, M, K, projs, P, num_sms, false)) != WL_OK) return st;
    out->grid = rp.ngroups * rp.c;
    out->cluster = rp.c;
    out->row_groups = rp.ngroups;
    out->nb_max = rp.nb_max;
    out->k_slice = rp.ks;
    out->smem_bytes = (long long)rp.smem;
    return WL_OK;
}

wl_status wl_last_device_status(void *stream) {
    std::lock_guard<std::mutex> lock(wl::g_mu);
    wl::DevicePool *pool = nullptr;
    wl_status st = wl::pool_for_current_device(&pool);
    if (st != WL_OK) return st;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return WL_ERR_CUDA;
    int word = 0;
    if (cudaMemcpy(&word, pool->words, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return WL_ERR_CUDA;
    // A kernel that gave up may have left its arrival counters set: clear the
    // whole word block (status and counters) after an error.
    if (word != 0 && cudaMemset(pool->words, 0, 64 * sizeof(int)) != cudaSuccess) return WL_ERR_CUDA;
    for (int slot : {(int)wl::kSlotTileCnt, (int)wl::kSlotFp4Cnt, (int)wl::kSlotFp4BCnt})
        if (word != 0 && pool->buf[slot] && cudaMemset(pool->buf[slot], 0, pool->cap[slot]) != cudaSuccess)
            return WL_ERR_CUDA;
    return static_cast<wl_status>(word);
}

wl_status wl_wait_probe(long long limit_ns, void *stream) {
    if (limit_ns <= 0 || limit_ns > 1000000000LL) return WL_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(wl::g_mu);
    wl::DevicePool *pool = nullptr;
    wl_status st = wl::pool_for_current_device(&pool);
    if (st != WL_OK) return st;
    return wl::from_cuda(wl::launch_wait_probe(pool->words + 1, pool->words,
                                               (unsigned long long)limit_ns,
                                               static_cast<cudaStream_t>(stream)));
}

int wl_version(void) { return (0 << 16) | 1; }

}  // extern "C"
