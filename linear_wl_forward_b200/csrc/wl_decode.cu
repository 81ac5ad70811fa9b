// Decode path (M <= 4 tokens): the memory-bound half of the theta-bundle
// linear, y = s (.) (W0 x) + U (V^T x).
//
// Two kernels, chained by programmatic dependent launch:
//
//  1. tvec_kernel: T = V^T x in fp32 (r x M per projection).  V is read once,
//     split over K across blocks; the last block of each projection to finish
//     adds the partial sums in block order (fixed order, no float atomics).
//     It releases the dependent grid immediately, so the decode kernel starts
//     streaming W0 while T is still being formed.
//
//  2. decode_kernel: one CTA per SM, each owning a balanced, contiguous range
//     of output rows.  A producer warp moves W0 row segments (2 KB each) into
//     an 8-deep shared-memory ring with 1-D bulk copies (TMA), completion
//     tracked by mbarriers; eight consumer warps each take one row per stage,
//     multiply it with the matching slice of x held in registers, reduce with
//     warp shuffles and keep z = W0 x per row in shared memory.  After the last
//     K panel, the ring streams the CTA's U rows; the consumers wait for T
//     (griddepcontrol.wait) and apply y = s * z + U_row . T in the epilogue, so
//     neither U V^T nor the low-rank product ever touches HBM.
//
// The design follows the custom-op kernel described on "Quality (Gemma 4
// 31B)", "Kernel optimizations", custom-op path (128-bit loads, warp-shuffle
// reductions, one warp per output row, cooperative V^T x, a single barrier),
// re-planned for sm_100a: bulk-copy staging replaces per-thread loads so one
// warp keeps 128 KB in flight per SM, and rows are split evenly across SMs.
#include "wl_common.cuh"
#include "wl_internal.h"

namespace wl {

// ------------------------------------------------------------- T = V^T x ---
template <int M>
__global__ void __launch_bounds__(256) tvec_kernel(const __grid_constant__ DecodeParams p) {
    // Let the decode kernel launch now: it only needs T in its epilogue and
    // waits for this grid there.
    pdl_launch_dependents();

    __shared__ float xs[M][kTChunk];
    __shared__ int s_last;

    const int b = blockIdx.x;
    int sp = 0;
    while (sp + 1 < p.nseg && b >= p.seg[sp + 1].tblk_begin) ++sp;
    const DecodeSeg &sg = p.seg[sp];
    const int r = sg.r;
    const int nblk = (p.K + kTChunk - 1) / kTChunk;
    const int c = b - sg.tblk_begin;
    const int k0 = c * kTChunk;
    const int kn = min(kTChunk, p.K - k0);

    for (int i = threadIdx.x; i < M * kTChunk; i += blockDim.x) {
        const int m = i / kTChunk, kk = i % kTChunk;
        xs[m][kk] = kk < kn ? __bfloat162float(p.x[(size_t)m * p.K + k0 + kk]) : 0.f;
    }
    __syncthreads();

    constexpr int kCols = WL_MAX_RANK / 256;
    float acc[M][kCols];
#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
        for (int q = 0; q < kCols; ++q) acc[m][q] = 0.f;

    const __nv_bfloat16 *Vb = sg.V + (size_t)k0 * r;
    for (int kk = 0; kk < kn; ++kk) {
#pragma unroll
        for (int q = 0; q < kCols; ++q) {
            const int j = threadIdx.x + q * 256;
            if (j < r) {
                const float v = __bfloat162float(Vb[(size_t)kk * r + j]);
#pragma unroll
                for (int m = 0; m < M; ++m) acc[m][q] = fmaf(v, xs[m][kk], acc[m][q]);
            }
        }
    }
    float *part = p.Tpart + (size_t)b * M * p.r_max;
#pragma unroll
    for (int q = 0; q < kCols; ++q) {
        const int j = threadIdx.x + q * 256;
        if (j < r) {
#pragma unroll
            for (int m = 0; m < M; ++m) part[(size_t)m * p.r_max + j] = acc[m][q];
        }
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(&p.counters[sp], 1) == nblk - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // Last block of this projection: add the partials in block order.
    for (int i = threadIdx.x; i < M * r; i += blockDim.x) {
        const int m = i / r, j = i % r;
        float t = 0.f;
        for (int cc = 0; cc < nblk; ++cc)
            t += __ldcg(p.Tpart + ((size_t)(sg.tblk_begin + cc) * M + m) * p.r_max + j);
        p.T[(size_t)m * p.t_ld + sg.t_off + j] = t;
    }
    if (threadIdx.x == 0) p.counters[sp] = 0;  // ready for the next call
}

// ---------------------------------------------------------------- decode ---
__device__ __forceinline__ int find_seg(const DecodeParams &p, int row) {
    int sp = 0;
    while (sp + 1 < p.nseg && row >= p.seg[sp + 1].row_begin) ++sp;
    return sp;
}

template <int M>
__device__ __forceinline__ void dot8_acc(const uint4 &w, const uint4 &xv, float &acc) {
    acc = fmaf(bf16lo(w.x), bf16lo(xv.x), acc);
    acc = fmaf(bf16hi(w.x), bf16hi(xv.x), acc);
    acc = fmaf(bf16lo(w.y), bf16lo(xv.y), acc);
    acc = fmaf(bf16hi(w.y), bf16hi(xv.y), acc);
    acc = fmaf(bf16lo(w.z), bf16lo(xv.z), acc);
    acc = fmaf(bf16hi(w.z), bf16hi(xv.z), acc);
    acc = fmaf(bf16lo(w.w), bf16lo(xv.w), acc);
    acc = fmaf(bf16hi(w.w), bf16hi(xv.w), acc);
}

template <int M>
__global__ void __launch_bounds__(kDecodeThreads, 1)
    decode_kernel(const __grid_constant__ DecodeParams p) {
    constexpr int KC = kDecodeKC;
    constexpr int NS = kDecodeStages;
    constexpr int RPS = kDecodeRowsPerStage;
    constexpr uint32_t kRowBytes = KC * 2;
    constexpr uint32_t kStageBytes = RPS * kRowBytes;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *ring = smem_raw;                                   // NS stages
    float *zpart = reinterpret_cast<float *>(ring + NS * kStageBytes);  // rows x M
    uint64_t *full = reinterpret_cast<uint64_t *>(zpart + kDecodeRowsCap * M);
    uint64_t *empty = full + NS;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + NS);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row_lo = (int)(((long long)blockIdx.x * p.total_rows) / gridDim.x);
    const int row_hi = (int)(((long long)(blockIdx.x + 1) * p.total_rows) / gridDim.x);
    const int K = p.K;
    const bool lowrank = p.has_lowrank != 0;
    const bool u_stream = lowrank && p.u_bulk;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], RPS);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == RPS) {
        // ------------------------------------------------ producer warp ----
        uint32_t it = 0;
        bool ok = true;
        for (int kc = 0; kc < K && ok; kc += KC) {
            const uint32_t kw = (uint32_t)min(KC, K - kc);
            for (int g = row_lo; g < row_hi; g += RPS) {
                const uint32_t slot = it % NS, ph = (it / NS) & 1u;
                if (!mbar_wait(&empty[slot], ph ^ 1u, p.status, p.timeout_ns) || *abort_flag) {
                    ok = false;
                    *abort_flag = 1;
                    break;
                }
                const int nr = min(RPS, row_hi - g);
                if (lane == 0) mbar_arrive_expect_tx(&full[slot], (uint32_t)nr * kw * 2u);
                __syncwarp();
                if (lane < nr) {
                    const int row = g + lane;
                    const DecodeSeg &sg = p.seg[find_seg(p, row)];
                    const __nv_bfloat16 *src = sg.W0 + (size_t)(row - sg.row_begin) * K + kc;
                    bulk_load(ring + slot * kStageBytes + lane * kRowBytes, src, kw * 2u, &full[slot]);
                }
                ++it;
            }
        }
        if (ok && u_stream) {
            for (int g = row_lo; g < row_hi; g += RPS) {
                const uint32_t slot = it % NS, ph = (it / NS) & 1u;
                if (!mbar_wait(&empty[slot], ph ^ 1u, p.status, p.timeout_ns) || *abort_flag) {
                    ok = false;
                    *abort_flag = 1;
                    break;
                }
                const int nr = min(RPS, row_hi - g);
                uint32_t bytes = 0;
                const __nv_bfloat16 *src = nullptr;
                if (lane < nr) {
                    const int row = g + lane;
                    const DecodeSeg &sg = p.seg[find_seg(p, row)];
                    bytes = (uint32_t)sg.r * 2u;
                    src = sg.U + (size_t)(row - sg.row_begin) * sg.r;
                }
                uint32_t total = bytes;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
                if (lane == 0) mbar_arrive_expect_tx(&full[slot], total);
                __syncwarp();
                if (bytes) bulk_load(ring + slot * kStageBytes + lane * kRowBytes, src, bytes, &full[slot]);
                ++it;
            }
        }
        if (!ok) {
            // Let copies already issued land before the CTA exits.
            const uint32_t inflight = it < (uint32_t)NS ? it : (uint32_t)NS;
            for (uint32_t i = it - inflight; i < it; ++i)
                mbar_wait(&full[i % NS], (i / NS) & 1u, p.status, 1000000ull);
        }
    } else {
        // ---------------------------------------------- consumer warps ----
        uint32_t it = 0;
        bool ok = true;
        for (int kc = 0; kc < K && ok; kc += KC) {
            uint4 xv[M][KC / 256];
#pragma unroll
            for (int m = 0; m < M; ++m)
#pragma unroll
                for (int j = 0; j < KC / 256; ++j) {
                    const int k = kc + j * 256 + lane * 8;
                    xv[m][j] = k < K ? __ldg(reinterpret_cast<const uint4 *>(p.x + (size_t)m * K + k))
                                     : make_uint4(0, 0, 0, 0);
                }
            for (int g = row_lo; g < row_hi; g += RPS) {
                const uint32_t slot = it % NS, ph = (it / NS) & 1u;
                if (!mbar_wait(&full[slot], ph, p.status, p.timeout_ns) || *abort_flag) {
                    ok = false;
                    *abort_flag = 1;
                    break;
                }
                const int row = g + warp;
                if (row < row_hi) {
                    const uint4 *wrow =
                        reinterpret_cast<const uint4 *>(ring + slot * kStageBytes + warp * kRowBytes);
                    float acc[M];
#pragma unroll
                    for (int m = 0; m < M; ++m) acc[m] = 0.f;
#pragma unroll
                    for (int j = 0; j < KC / 256; ++j) {
                        if (kc + j * 256 + lane * 8 < K) {
                            const uint4 w = wrow[j * 32 + lane];
#pragma unroll
                            for (int m = 0; m < M; ++m) dot8_acc<M>(w, xv[m][j], acc[m]);
                        }
                    }
#pragma unroll
                    for (int m = 0; m < M; ++m) acc[m] = warp_sum(acc[m]);
                    if (lane == 0) {
                        float *zp = zpart + (row - row_lo) * M;
#pragma unroll
                        for (int m = 0; m < M; ++m) zp[m] = (kc == 0 ? 0.f : zp[m]) + acc[m];
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[slot]);
                ++it;
            }
        }

        if (ok) {
            // ------------------------------------------------- epilogue ----
            if (lowrank) pdl_wait_primary();  // T = V^T x is complete and visible
            for (int g = row_lo; g < row_hi; g += RPS) {
                uint32_t slot = 0;
                if (u_stream) {
                    slot = it % NS;
                    const uint32_t ph = (it / NS) & 1u;
                    if (!mbar_wait(&full[slot], ph, p.status, p.timeout_ns) || *abort_flag) {
                        *abort_flag = 1;
                        break;
                    }
                }
                const int row = g + warp;
                if (row < row_hi) {
                    const int sp = find_seg(p, row);
                    const DecodeSeg &sg = p.seg[sp];
                    const int local = row - sg.row_begin;
                    float acc[M];
#pragma unroll
                    for (int m = 0; m < M; ++m) acc[m] = 0.f;
                    if (sg.r > 0) {
                        const float *T = p.T + sg.t_off;
                        if (u_stream) {
                            const uint4 *urow = reinterpret_cast<const uint4 *>(
                                ring + slot * kStageBytes + warp * kRowBytes);
                            for (int j0 = lane * 8; j0 < sg.r; j0 += 256) {
                                const uint4 u = urow[j0 / 8];
#pragma unroll
                                for (int m = 0; m < M; ++m) {
                                    const float4 t0 = __ldcg(reinterpret_cast<const float4 *>(
                                        T + (size_t)m * p.t_ld + j0));
                                    const float4 t1 = __ldcg(reinterpret_cast<const float4 *>(
                                        T + (size_t)m * p.t_ld + j0 + 4));
                                    float a = acc[m];
                                    a = fmaf(bf16lo(u.x), t0.x, a);
                                    a = fmaf(bf16hi(u.x), t0.y, a);
                                    a = fmaf(bf16lo(u.y), t0.z, a);
                                    a = fmaf(bf16hi(u.y), t0.w, a);
                                    a = fmaf(bf16lo(u.z), t1.x, a);
                                    a = fmaf(bf16hi(u.z), t1.y, a);
                                    a = fmaf(bf16lo(u.w), t1.z, a);
                                    a = fmaf(bf16hi(u.w), t1.w, a);
                                    acc[m] = a;
                                }
                            }
                        } else {
                            const __nv_bfloat16 *urow = sg.U + (size_t)local * sg.r;
                            for (int j = lane; j < sg.r; j += 32) {
                                const float u = __bfloat162float(urow[j]);
#pragma unroll
                                for (int m = 0; m < M; ++m)
                                    acc[m] = fmaf(u, __ldcg(T + (size_t)m * p.t_ld + j), acc[m]);
                            }
                        }
#pragma unroll
                        for (int m = 0; m < M; ++m) acc[m] = warp_sum(acc[m]);
                    }
                    if (lane == 0) {
                        const float sc = sg.s[local];
                        const float *zp = zpart + (row - row_lo) * M;
#pragma unroll
                        for (int m = 0; m < M; ++m)
                            sg.y[(size_t)m * sg.N + local] = __float2bfloat16_rn(fmaf(sc, zp[m], acc[m]));
                    }
                }
                if (u_stream) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[slot]);
                    ++it;
                }
            }
        }
    }
    __syncthreads();
}

size_t decode_smem_bytes(int M) {
    return (size_t)kDecodeStages * kDecodeRowsPerStage * kDecodeKC * 2 +
           (size_t)kDecodeRowsCap * M * sizeof(float) + 2 * kDecodeStages * sizeof(uint64_t) + 16;
}

int decode_t_blocks(int K) { return (K + kTChunk - 1) / kTChunk; }

template <int M>
static cudaError_t launch_decode_m(const DecodeParams &p, int num_sms, cudaStream_t stream) {
    const size_t smem = decode_smem_bytes(M);
    // Opt in to the large shared-memory carve-out once per device.
    static bool attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_done[dev]) {
        e = cudaFuncSetAttribute(decode_kernel<M>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }

    if (p.has_lowrank) {
        int tblocks = 0;
        for (int i = 0; i < p.nseg; ++i)
            if (p.seg[i].r > 0) tblocks = p.seg[i].tblk_begin + decode_t_blocks(p.K);
        tvec_kernel<M><<<tblocks, 256, 0, stream>>>(p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }

    int grid = (p.total_rows + kDecodeRowsPerStage - 1) / kDecodeRowsPerStage;
    if (grid > num_sms) grid = num_sms;
    const int min_grid = (p.total_rows + kDecodeRowsCap - 1) / kDecodeRowsCap;
    if (grid < min_grid) grid = min_grid;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kDecodeThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    if (p.has_lowrank) {
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, decode_kernel<M>, p);
}

cudaError_t launch_decode(const DecodeParams &p, int num_sms, cudaStream_t stream) {
    switch (p.M) {
        case 1: return launch_decode_m<1>(p, num_sms, stream);
        case 2: return launch_decode_m<2>(p, num_sms, stream);
        case 3: return launch_decode_m<3>(p, num_sms, stream);
        case 4: return launch_decode_m<4>(p, num_sms, stream);
        default: return cudaErrorInvalidValue;
    }
}

// ----------------------------------------------------------- wait probe ----
__global__ void wait_probe_kernel(volatile int *flag, int *status, unsigned long long limit_ns) {
    const uint64_t t0 = globaltimer_ns();
    while (*flag == 0) {
        if (globaltimer_ns() - t0 > limit_ns) {
            record_status(status, kStatusTimeout);
            return;
        }
        __nanosleep(1000);
    }
}

cudaError_t launch_wait_probe(int *flag, int *status, unsigned long long limit_ns,
                              cudaStream_t stream) {
    wait_probe_kernel<<<1, 1, 0, stream>>>(flag, status, limit_ns);
    return cudaGetLastError();
}

}  // namespace wl
