// Tensor-core path (any M; see wl_path for when it is chosen): a persistent
// tcgen05 GEMM whose epilogue applies the per-row scale and adds the rank-r
// term,
//
//     y[m][n] = s[n] * sum_k x[m][k] W0[n][k]  +  sum_j T[m][j] U[n][j],
//     T = x V (computed first by the same kernel in plain mode, bf16 output).
//
// Per CTA (one per SM, 192 threads):
//   warp 0      TMA producer: 128 x 64 tiles of x (or T) and BN x 64 tiles of
//               W0 (or U), 128-byte swizzled, into a 4-deep ring of 48 KB
//               stages, completion on mbarriers (no multicast).
//   warp 1      allocates 512 TMEM columns; one lane issues tcgen05.mma
//               (128 x BN x 16, bf16 in, fp32 accumulate): the K loop over W0
//               into accumulator A, then the r/64 low-rank blocks into
//               accumulator B.  With BN = 256 the two fill TMEM (A at column
//               0, B at 256) and the next tile's MMAs wait for the epilogue;
//               narrower tiles (and the swap mode) keep two sets of [A | B]
//               (columns 0 and 256) and alternate, so the next tile's MMAs
//               run while the epilogue drains the last.  (256-column tiles
//               stay the faster choice for prefill: 1116 TFLOP/s single-set
//               against 815 with 128-column double-set tiles on the Gemma-4
//               gate/up call.)  Each stage is released with tcgen05.commit;
//               the finished tile is signalled to the epilogue the same way.
//   warps 2-5   epilogue: tcgen05.ld of both accumulators (one TMEM lane = one
//               token row per thread), y = s * A + B in fp32, one rounding to
//               bf16, stores with edge checks.
// The scale touches only the shared-block product, so the two products keep
// separate accumulators; U V^T is never formed.
//
// Swap-AB mode (few tokens, M <= 16): the 128-row side of the MMA runs over
// output rows instead -- A = 128 x 64 tiles of W0 (then U), B = x (then T)
// tiles of mp = M rounded up to 16 rows, D = 128 rows x mp tokens -- so a
// tile streams 128 full rows of W0 and no MMA lanes are spent on absent
// tokens.  When the output rows alone give fewer tiles than SMs, K is cut
// into ranges (at most 8, each >= 8 blocks) whose sums are stored; the CTA
// that completes a tile's arrival count adds them up in range order
// (deterministic) and writes y.
//
// Bf16 operands with fp32 accumulation follow "Quality (Gemma 4 31B)", "Kernel
// optimizations", GEMM path item 2 (bf16 matmuls accumulate in fp32 on the
// tensor cores); the pages' GEMM path uses two library matmuls per stack, here
// the low-rank product rides in the same kernel and the same accumulator pass.
#include <atomic>

#include "wl_common.cuh"
#include "wl_internal.h"
#include "wl_prefetch.cuh"

namespace wl {

namespace {

// Launch with programmatic dependent launch: the kernel may start while the
// previous kernel in the stream finishes; each kernel here waits for it
// (griddepcontrol.wait) before its first global-memory access.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

constexpr uint32_t kABytes = kGemmBM * kGemmBK * 2;     // 16 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccBCol = 256;

struct TileInfo {
    int seg, m0, n0;
};

__device__ __forceinline__ TileInfo tile_info(const GemmParams &p, int t) {
    int sp = 0;
    while (sp + 1 < p.nseg && t >= p.seg[sp + 1].tile_begin) ++sp;
    const int local = t - p.seg[sp].tile_begin;
    TileInfo ti;
    ti.seg = sp;
    ti.m0 = (local % p.num_m_tiles) * kGemmBM;
    ti.n0 = (local / p.num_m_tiles) * p.BN;
    return ti;
}

// All lanes wait; the warp agrees on the outcome.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, const GemmParams &p,
                                          volatile int *abort_flag) {
    bool ok = mbar_wait(bar, parity, p.status, p.timeout_ns) && (*abort_flag == 0);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && (threadIdx.x & 31) == 0) *abort_flag = 1;
    return ok;
}

}  // namespace

__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(const __grid_constant__ GemmParams p) {
    // The next kernel may launch now; it waits for this grid before touching
    // memory.  This grid's own global accesses start after the wait below.
    pdl_launch_dependents();
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    uint8_t *base = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    const uint32_t stages = (uint32_t)p.stages, stage_bytes = (uint32_t)p.stage_bytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(base + stages * stage_bytes);
    uint64_t *empty = full + stages;
    uint64_t *tmem_full = empty + stages;  // [2]
    uint64_t *tmem_empty = tmem_full + 2;  // [2]
    uint64_t *drain = tmem_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *last_flag = abort_flag + 1;  // swap mode: this CTA adds up the tile's K ranges

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nkb = (p.K + kGemmBK - 1) / kGemmBK;
    // Operand B rows per stage: W0 / U tiles of BN rows, or (swap) x / T
    // tiles of mp rows; operand A is always 128 rows (x / T, or W0 / U).
    const uint32_t b_rows = p.swap ? (uint32_t)p.mp : (uint32_t)p.BN;
    const uint32_t b_bytes = b_rows * kGemmBK * 2;
    const int units = p.num_tiles * p.ksplit;
    // TMEM accumulators.  Tiles of at most 128 columns (and the swap mode's
    // token tiles) use two sets, [A | B] at columns 0 and 256, so the MMAs of
    // the next tile run while the epilogue drains this one; 256-column tiles
    // use one set (A at 0, B at 256) and the MMAs wait for the drain.
    const bool dbuf = p.swap || p.BN <= 128;
    const uint32_t acc_b = dbuf ? 128u : kAccBCol;  // B's offset inside a set
    auto acc_set = [&](uint32_t tc) -> uint32_t { return dbuf ? (tc & 1u) : 0u; };
    auto acc_phase = [&](uint32_t tc) -> uint32_t { return dbuf ? (tc >> 1) & 1u : tc & 1u; };

    if (threadIdx.x == 0) {
        for (uint32_t i = 0; i < stages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tmem_full[i], 1);
            mbar_init(&tmem_empty[i], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&p.tm_a);
        prefetch_tmap(&p.tm_t);
        for (int i = 0; i < p.nseg; ++i) {
            prefetch_tmap(&p.tm_b[i]);
            prefetch_tmap(&p.tm_u[i]);
        }
        l2_prefetch_share(p.pf, blockIdx.x, gridDim.x);  // the following call's weights
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait_primary();  // the previous kernel is done: x, T and the scratch are ours

    if (warp == 0) {
        // ------------------------------------------------------ producer ----
        uint32_t it = 0, slot = 0, ph = 0;  // ring position, tracked without divisions
        bool ok = true;
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            const int tile = u / p.ksplit, split = u - tile * p.ksplit;
            const TileInfo ti = tile_info(p, tile);
            const GemmSeg &sg = p.seg[ti.seg];
            const int kb0 = split * p.kb_split;
            const int kb1 = min(nkb, kb0 + p.kb_split);
            const int lr = split == 0 ? sg.lr_blocks : 0;
            const int total = (kb1 - kb0) + lr;
            for (int i = 0; i < total; ++i) {
                if (!warp_wait(&empty[slot], ph ^ 1u, p, abort_flag)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    uint8_t *sa = base + slot * stage_bytes;
                    uint8_t *sb = sa + kABytes;
                    mbar_arrive_expect_tx(&full[slot], kABytes + b_bytes);
                    if (i < kb1 - kb0) {
                        const int kc = (kb0 + i) * kGemmBK;
                        if (p.swap) {
                            tma_load_2d(sa, &p.tm_b[ti.seg], kc, ti.n0, &full[slot]);
                            tma_load_2d(sb, &p.tm_a, kc, 0, &full[slot]);
                        } else {
                            tma_load_2d(sa, &p.tm_a, kc, ti.m0, &full[slot]);
                            tma_load_2d(sb, &p.tm_b[ti.seg], kc, ti.n0, &full[slot]);
                        }
                    } else {
                        const int j0 = (i - (kb1 - kb0)) * kGemmBK;
                        if (p.swap) {
                            tma_load_2d(sa, &p.tm_u[ti.seg], j0, ti.n0, &full[slot]);
                            tma_load_2d(sb, &p.tm_t, sg.t_col + j0, 0, &full[slot]);
                        } else {
                            tma_load_2d(sa, &p.tm_t, sg.t_col + j0, ti.m0, &full[slot]);
                            tma_load_2d(sb, &p.tm_u[ti.seg], j0, ti.n0, &full[slot]);
                        }
                    }
                }
                __syncwarp();
                ++it;
                if (++slot == stages) {
                    slot = 0;
                    ph ^= 1u;
                }
            }
        }
        if (!ok) {
            // Let the loads already issued land before the CTA exits.
            const uint32_t inflight = it < stages ? it : stages;
            for (uint32_t i = it - inflight; i < it; ++i)
                mbar_wait(&full[i % stages], (i / stages) & 1u, p.status, 1000000ull);
        }
    } else if (warp == 1) {
        // ----------------------------------------------------- MMA issuer ---
        const uint32_t idesc = idesc_bf16_f32(kGemmBM, b_rows);
        uint32_t slot = 0, ph = 0, tcount = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            const int tile = u / p.ksplit, split = u - tile * p.ksplit;
            const TileInfo ti = tile_info(p, tile);
            const GemmSeg &sg = p.seg[ti.seg];
            const int kb0 = split * p.kb_split;
            const int nmain = min(nkb, kb0 + p.kb_split) - kb0;
            const int total = nmain + (split == 0 ? sg.lr_blocks : 0);
            const uint32_t set = acc_set(tcount);
            if (!warp_wait(&tmem_empty[set], acc_phase(tcount) ^ 1u, p, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            for (int i = 0; i < total; ++i) {
                if (!warp_wait(&full[slot], ph, p, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t a_addr = smem_addr(base + slot * stage_bytes);
                    const uint32_t b_addr = a_addr + kABytes;
                    const uint64_t adesc = sw128_kmajor_desc(a_addr);
                    const uint64_t bdesc = sw128_kmajor_desc(b_addr);
                    const bool lowrank = i >= nmain;
                    const uint32_t d = tmem_base + set * 256u + (lowrank ? acc_b : 0u);
                    const bool first = (i == 0) || (i == nmain);
#pragma unroll
                    for (int k = 0; k < kGemmBK / 16; ++k) {
                        // advance 16 elements (32 bytes) along K inside the swizzle row
                        tc_mma_f16(d, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), idesc,
                                   (first && k == 0) ? 0u : 1u);
                    }
                    tc_commit(&empty[slot]);
                }
                __syncwarp();
                if (++slot == stages) {
                    slot = 0;
                    ph ^= 1u;
                }
            }
            if (!ok) break;
            if (lane == 0) tc_commit(&tmem_full[set]);
            __syncwarp();
            ++tcount;
        }
        if (!ok) {
            // Wait for MMAs already issued before TMEM is released.
            if (lane == 0) tc_commit(drain);
            __syncwarp();
            mbar_wait(drain, 0, p.status, 1000000ull);
        }
    } else if (!p.swap) {
        // ------------------------------------------------------- epilogue ---
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int row_in_tile = q * 32 + lane;
        const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16);
        uint32_t tcount = 0;
        for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
            const TileInfo ti = tile_info(p, t);
            const GemmSeg &sg = p.seg[ti.seg];
            const uint32_t set = acc_set(tcount);
            if (!warp_wait(&tmem_full[set], acc_phase(tcount), p, abort_flag)) break;
            tc_fence_after();
            const uint32_t acc_addr = lane_addr + set * 256u;
            const int m = ti.m0 + row_in_tile;
            const bool lr = sg.lr_blocks > 0;
            const bool vec = ((reinterpret_cast<uintptr_t>(sg.y) & 15u) == 0) && (sg.ldy % 8 == 0);
            __nv_bfloat16 *yrow = sg.y + (size_t)m * sg.ldy;
            for (int c = 0; c < p.BN; c += 32) {
                uint32_t a[32], b[32];
                tmem_ld32(acc_addr + (uint32_t)c, a);
                if (lr) tmem_ld32(acc_addr + acc_b + (uint32_t)c, b);
                tmem_ld_wait();
                const int nb = ti.n0 + c;
                if (m < p.M && nb < sg.N) {
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int n = nb + i;
                        const float sc = (sg.s && n < sg.N) ? __ldg(sg.s + n) : 1.f;
                        const float acc = __uint_as_float(a[i]);
                        v[i] = lr ? fmaf(sc, acc, __uint_as_float(b[i])) : sc * acc;
                    }
                    if (vec && nb + 32 <= sg.N) {
                        uint4 *dst = reinterpret_cast<uint4 *>(yrow + nb);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            uint4 w;
                            w.x = pack_bf16x2(v[8 * i + 0], v[8 * i + 1]);
                            w.y = pack_bf16x2(v[8 * i + 2], v[8 * i + 3]);
                            w.z = pack_bf16x2(v[8 * i + 4], v[8 * i + 5]);
                            w.w = pack_bf16x2(v[8 * i + 6], v[8 * i + 7]);
                            dst[i] = w;
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (nb + i < sg.N) yrow[nb + i] = __float2bfloat16_rn(v[i]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tmem_empty[set]);
            ++tcount;
        }
    } else {
        // ------------------------------------------------- swap epilogue ---
        // TMEM lane = output row n0 + lane_in_tile, column = token.  With one
        // K range per tile: y = s * A + B directly.  With several: each range
        // stores its sums; the CTA that completes a tile's arrival count adds
        // the ranges up in range order (deterministic) and writes y.  The four
        // epilogue warps then meet at named barriers, so they also decide
        // together to stop (bar.red.or) -- none may leave one alone.
        const int q = warp & 3;
        const int row_in_tile = q * 32 + lane;
        const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16);
        const int mp = p.mp;
        const size_t tile_stride = (size_t)mp * kGemmBM;
        uint32_t tcount = 0;
        for (int u = blockIdx.x; u < units; u += gridDim.x) {
            const int tile = u / p.ksplit, split = u - tile * p.ksplit;
            const TileInfo ti = tile_info(p, tile);
            const GemmSeg &sg = p.seg[ti.seg];
            const uint32_t set = acc_set(tcount);
            bool ok = warp_wait(&tmem_full[set], acc_phase(tcount), p, abort_flag);
            if (p.ksplit > 1) {
                uint32_t any_fail;
                asm volatile(
                    "{\n\t.reg .pred p, q;\n\t"
                    "setp.ne.u32 p, %1, 0;\n\t"
                    "bar.red.or.pred q, 1, 128, p;\n\t"
                    "selp.u32 %0, 1, 0, q;\n\t}"
                    : "=r"(any_fail)
                    : "r"((uint32_t)!ok)
                    : "memory");
                ok = any_fail == 0;
            }
            if (!ok) break;
            tc_fence_after();
            const int n = ti.n0 + row_in_tile;
            const bool lr = sg.lr_blocks > 0;
            const bool lr_here = lr && split == 0;
            const float sc = (sg.s && n < sg.N) ? __ldg(sg.s + n) : 1.f;
            float *zp = p.part + ((size_t)split * p.num_tiles + tile) * tile_stride + row_in_tile;
            float *dp = p.part + ((size_t)p.ksplit * p.num_tiles + tile) * tile_stride + row_in_tile;
            for (int c = 0; c < mp; c += 32) {
                uint32_t a[32], b[32];
                tmem_ld32(lane_addr + set * 256u + (uint32_t)c, a);
                if (lr_here) tmem_ld32(lane_addr + set * 256u + acc_b + (uint32_t)c, b);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int m = c + i;
                    if (m >= p.M) break;
                    const float za = __uint_as_float(a[i]);
                    const float zb = lr_here ? __uint_as_float(b[i]) : 0.f;
                    if (p.ksplit == 1) {
                        if (n < sg.N) sg.y[(size_t)m * sg.ldy + n] = __float2bfloat16_rn(fmaf(sc, za, zb));
                    } else {
                        // [split][tile][token][row] partial sums, rows contiguous
                        zp[(size_t)m * kGemmBM] = za;
                        if (lr_here) dp[(size_t)m * kGemmBM] = zb;
                    }
                }
            }
            // TMEM is read: the MMA warp may reuse this set.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tmem_empty[set]);
            ++tcount;
            if (p.ksplit == 1) continue;
            __threadfence();
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (warp == 2 && lane == 0)
                *last_flag = atomicAdd(&p.tile_cnt[tile], 1u) == (unsigned)(p.ksplit - 1) ? 1 : 0;
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (*last_flag) {
                __threadfence();
                if (n < sg.N) {
                    // eight tokens at a time, every range's value loaded before
                    // any is added (independent loads), then added in range order
                    const float *zr = p.part + (size_t)tile * tile_stride + row_in_tile;
                    const size_t split_stride = (size_t)p.num_tiles * tile_stride;
                    for (int m0 = 0; m0 < p.M; m0 += 8) {
                        float v[kGemmMaxKSplit][8], d[8];
#pragma unroll
                        for (int sidx = 0; sidx < kGemmMaxKSplit; ++sidx)
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                v[sidx][i] = (sidx < p.ksplit && m0 + i < p.M)
                                                 ? __ldcg(zr + sidx * split_stride + (size_t)(m0 + i) * kGemmBM)
                                                 : 0.f;
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            d[i] = (lr && m0 + i < p.M) ? __ldcg(dp + (size_t)(m0 + i) * kGemmBM) : 0.f;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            if (m0 + i >= p.M) break;
                            float z = 0.f;
#pragma unroll
                            for (int sidx = 0; sidx < kGemmMaxKSplit; ++sidx) z += v[sidx][i];
                            sg.y[(size_t)(m0 + i) * sg.ldy + n] = __float2bfloat16_rn(fmaf(sc, z, d[i]));
                        }
                    }
                }
                if (warp == 2 && lane == 0) p.tile_cnt[tile] = 0u;  // for the next call
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");  // last_flag is reused by the next unit
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// Pipeline depth for the tile shapes: stages of a 128 x 64 A tile and a
// BN x 64 (or, swap, mp x 64) B tile, as many as fit in 200 KB (at most
// kGemmMaxStages).
void set_gemm_stages(GemmParams &p) {
    const uint32_t b_rows = p.swap ? (uint32_t)p.mp : (uint32_t)p.BN;
    p.stage_bytes = (int)(kABytes + b_rows * kGemmBK * 2);  // multiples of 1024 (rows % 8 == 0)
    int n = (200 * 1024) / p.stage_bytes;
    p.stages = n > kGemmMaxStages ? kGemmMaxStages : (n < 2 ? 2 : n);
}

size_t gemm_smem_bytes(const GemmParams &p) {
    return 1024 + (size_t)p.stages * p.stage_bytes + (2 * kGemmMaxStages + 5) * 8 + 16;
}

cudaError_t launch_gemm(const GemmParams &p, int num_sms, cudaStream_t stream) {
    const size_t smem = gemm_smem_bytes(p);
    if (p.stages < 2 || p.stages > kGemmMaxStages || smem > 227 * 1024) return cudaErrorInvalidValue;
    // Opt in to the large shared-memory carve-out once per device.
    static std::atomic<bool> attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_done[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        attr_done[dev].store(true, std::memory_order_release);
    }
    if (p.ksplit < 1 || (p.swap && (p.mp < 16 || p.mp > 64 || p.mp % 16 != 0))) return cudaErrorInvalidValue;
    const int units = p.num_tiles * p.ksplit;
    int grid = units < num_sms ? units : num_sms;
    if (grid < 1) return cudaSuccess;
    return launch_pdl(gemm_kernel, dim3(grid), dim3(kGemmThreads), smem, stream, p);
}

// ---------------------------------------------------------- small helpers ---
// Vt rows of every projection of a call (blockIdx.z = projection).
__global__ void transpose_v_kernel(const __grid_constant__ TransposeVArgs a) {
    pdl_launch_dependents();
    pdl_wait_primary();
    const int pi = blockIdx.z;
    const __nv_bfloat16 *__restrict__ V = a.V[pi];
    const int K = a.K, r = a.r[pi], r_pad = a.r_pad[pi];
    __nv_bfloat16 *__restrict__ Vt = a.Vt + (size_t)a.row[pi] * K;
    __shared__ __nv_bfloat16 tile[32][33];
    const int k0 = blockIdx.x * 32, j0 = blockIdx.y * 32;
    if (j0 >= r_pad) return;
    const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
    for (int i = ty; i < 32; i += 8) {
        const int k = k0 + i, j = j0 + tx;
        tile[i][tx] = (k < K && j < r) ? V[(size_t)k * r + j] : __float2bfloat16_rn(0.f);
    }
    __syncthreads();
    for (int i = ty; i < 32; i += 8) {
        const int j = j0 + i, k = k0 + tx;
        if (j < r_pad && k < K) Vt[(size_t)j * K + k] = tile[tx][i];
    }
}

cudaError_t launch_transpose_v(const TransposeVArgs &a, cudaStream_t stream) {
    if (a.n < 1 || a.n > kMaxSeg) return cudaErrorInvalidValue;
    int max_rpad = 0;
    for (int i = 0; i < a.n; ++i) max_rpad = a.r_pad[i] > max_rpad ? a.r_pad[i] : max_rpad;
    dim3 grid((a.K + 31) / 32, (max_rpad + 31) / 32, a.n);
    return launch_pdl(transpose_v_kernel, grid, dim3(32, 8), 0, stream, a);
}

__global__ void pad_u_kernel(const __nv_bfloat16 *__restrict__ U, int N, int r, int r_pad,
                             __nv_bfloat16 *__restrict__ Upad) {
    pdl_launch_dependents();
    pdl_wait_primary();
    const size_t total = (size_t)N * r_pad;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
         i += (size_t)gridDim.x * blockDim.x) {
        const size_t n = i / r_pad;
        const int j = (int)(i % r_pad);
        Upad[i] = j < r ? U[n * r + j] : __float2bfloat16_rn(0.f);
    }
}

cudaError_t launch_pad_u(const __nv_bfloat16 *U, int N, int r, int r_pad, __nv_bfloat16 *Upad,
                         cudaStream_t stream) {
    const size_t total = (size_t)N * r_pad;
    int blocks = (int)((total + 255) / 256);
    if (blocks > 4096) blocks = 4096;
    if (blocks < 1) return cudaSuccess;
    return launch_pdl(pad_u_kernel, dim3(blocks), dim3(256), 0, stream, U, N, r, r_pad, Upad);
}

}  // namespace wl
