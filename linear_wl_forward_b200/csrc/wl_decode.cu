// Decode path (M <= 16 tokens): the memory-bound half of the theta-bundle
// linear, y = s (.) (W0 x) + U (V^T x), as ONE kernel per call.
//
// Work split: the output rows of the (stacked) call are cut into blocks of 16
// rows that never straddle two projections; each CTA (one per SM at most) owns
// a balanced, contiguous range of blocks.  For every block, each of the eight
// consumer warps takes a fixed 1/8 share of the 64-column chunks of K (and of
// the rank r), so all warps stream the same number of bytes.
//
// Roles (nine warps):
//  * producer warp: for each block and each consumer warp, moves the 16 rows x
//    (up to) 256 columns of W0 -- then of U -- that the warp needs into one of
//    that warp's two 8 KB shared-memory slots with TMA tensor copies (a single
//    3-D box {64 columns, 16 rows, 4 chunks} per full slot, 128-byte swizzle,
//    no multicast), completion counted on mbarriers; 16 slots keep up to 128 KB
//    in flight per SM.  W0 and U are parameters, so the producer starts at
//    once, also while the previous kernel in the stream is still running
//    (programmatic dependent launch).  Rows past the end of a projection are
//    out of bounds for the copy and arrive as zeros.
//  * consumer warps: wait for the previous kernel (griddepcontrol.wait: x and
//    the scratch become valid), form T = V^T x (below), then for each slot run
//    warp-level tensor-core MMAs (m16n8k16, bf16 in, fp32 accumulate): A = the
//    16 W0 rows read with ldmatrix through the swizzle (conflict-free), B = x
//    (token n, column k) loaded from L1/L2.  The U slots go through a second
//    accumulator with B = T split into bf16 high and low parts, so the
//    low-rank product keeps fp32-level accuracy.  At the end of a block the
//    eight warps' accumulators are added in warp order in shared memory and
//    y = s * (W0 x) + U T is rounded once to bf16.
//
// T = V^T x is formed inside the same kernel ("cooperative vtx" of the pages'
// custom op), one of two ways chosen per call on the host:
//  * local: when every CTA's share of V is small (<= 96 KB), each CTA reads the
//    V slices its rows need (from L2 after the first touch) and reduces them in
//    shared memory;
//  * grid: otherwise each CTA forms partial sums over a 1/grid slice of K for
//    every projection and writes them to scratch; after a grid-wide arrival
//    count (a bounded wait), CTA c adds up column block c of T over all CTAs
//    (lanes stride the CTAs, then a fixed shuffle tree); after a second count
//    every CTA loads the T slices its rows need.  The counters reset
//    themselves once every CTA is past both counts.
// Every sum has a fixed order (no float atomics), so results are reproducible.
//
// Prior art: the custom-op kernel on "Quality (Gemma 4 31B)", "Kernel
// optimizations", custom-op path (128-bit loads, warp-shuffle reductions, one
// warp per output row, cooperative V^T x, a single block barrier).  Here the
// W0 stream is staged by TMA, the per-row dot products run on the tensor cores
// (the stream stays HBM-bound and the instruction count per byte drops by an
// order of magnitude), rows are spread evenly over all SMs, and consecutive
// calls overlap through PDL.
#include "wl_common.cuh"
#include "wl_internal.h"

namespace wl {

namespace {

constexpr int NW = kDecodeWarps;
constexpr int BR = kDecodeBlockRows;
constexpr int CK = kDecodeChunkK;
constexpr int SC = kDecodeSlotChunks;
constexpr int SLOTS = kDecodeSlotsPerWarp;
constexpr size_t kLocalVBytes = 96 * 1024;
constexpr uint32_t kDecodeMaxSmem = 227 * 1024;

__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kDecodeConsumers) : "memory");
}

// Barrier over the 256 consumer threads that also ORs a predicate across them,
// so every consumer takes the same abort decision.
__device__ __forceinline__ bool consumer_any(bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out)
        : "r"((uint32_t)pred), "n"(kDecodeConsumers)
        : "memory");
    return out != 0;
}

__device__ __forceinline__ unsigned int ld_acquire_gpu(const unsigned int *p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_gpu_add(unsigned int *p, unsigned int v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Arrive on a grid-wide counter and wait (bounded) until all CTAs arrived.
__device__ __forceinline__ bool grid_arrive_wait(unsigned int *ctr, unsigned int expected,
                                                 const DecodeParams &p) {
    red_release_gpu_add(ctr, 1u);
    const uint64_t t0 = globaltimer_ns();
    uint32_t polls = 0;
    while (ld_acquire_gpu(ctr) < expected) {
        if ((++polls & 63u) == 0 && globaltimer_ns() - t0 > p.timeout_ns) {
            record_status(p.status, kStatusTimeout);
            return false;
        }
    }
    return true;
}

// Block b of the call: its projection, first row within it and row count.
struct Block {
    int sp, row0, nrows;
};

__device__ __forceinline__ Block block_info(const DecodeParams &p, int b) {
    int sp = 0;
    while (sp + 1 < p.nseg && b >= p.seg[sp + 1].blk_begin) ++sp;
    Block B;
    B.sp = sp;
    B.row0 = (b - p.seg[sp].blk_begin) * BR;
    B.nrows = min(BR, p.seg[sp].N - B.row0);
    return B;
}

__device__ __forceinline__ int seg_blocks(const DecodeSeg &sg) { return (sg.N + BR - 1) / BR; }

__device__ __forceinline__ bool seg_touched(const DecodeSeg &sg, int blk_lo, int blk_hi) {
    return sg.r > 0 && sg.blk_begin < blk_hi && sg.blk_begin + seg_blocks(sg) > blk_lo;
}

// All lanes wait on the barrier phase; the warp agrees on the outcome.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, const DecodeParams &p,
                                          volatile int *abort_flag) {
    bool ok = mbar_wait(bar, parity, p.status, p.timeout_ns) && (*abort_flag == 0);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && (threadIdx.x & 31) == 0) *abort_flag = 1;
    return ok;
}

__device__ __forceinline__ void tma_load_3d(void *dst_smem, const void *tmap, int c0, int c1, int c2,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_addr(dst_smem)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t (&a)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                 : "r"(addr));
}

// D += A(16x16, row) * B(16x8, col), bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7},"
        " {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t ldg_u32(const __nv_bfloat16 *p) {
    return __ldg(reinterpret_cast<const unsigned int *>(p));
}

// Chunks [lo, hi) of consumer warp w among n chunks.
__device__ __forceinline__ void warp_chunks(int n, int w, int &lo, int &hi) {
    lo = (w * n) / NW;
    hi = ((w + 1) * n) / NW;
}

// Chunks of the rank r that warp w streams: handed out in reverse warp order,
// so they land first on the warps whose W0 share is one chunk short.
__device__ __forceinline__ void warp_u_chunks(int r, int w, int &lo, int &hi) {
    warp_chunks((r + CK - 1) / CK, NW - 1 - w, lo, hi);
}

// A warp's position in its sequence of ring copies: slot s of block b, with
// the block's layout for this warp (W0 chunks are fixed for the call, U chunks
// depend on the block's projection).
struct WarpSeq {
    int b, s;
    int ns, nw0;       // slots in this block, of which W0 slots
    int u_lo, u_hi;    // U chunk range in this block
    int sp, row0, nrows;
};

__device__ __forceinline__ void seq_load(const DecodeParams &p, int w, int w0_slots, WarpSeq &q) {
    const Block B = block_info(p, q.b);
    q.sp = B.sp;
    q.row0 = B.row0;
    q.nrows = B.nrows;
    q.nw0 = w0_slots;
    q.u_lo = q.u_hi = 0;
    const int r = p.seg[B.sp].r;
    if (p.u_bulk && r > 0) warp_u_chunks(r, w, q.u_lo, q.u_hi);
    q.ns = w0_slots + (q.u_hi - q.u_lo + SC - 1) / SC;
}

// Moves q to the next slot this warp streams, crossing blocks as needed;
// false once the CTA's blocks are exhausted.
__device__ __forceinline__ bool seq_next(const DecodeParams &p, int w, int w0_slots, int blk_hi,
                                         WarpSeq &q) {
    ++q.s;
    while (q.s >= q.ns) {
        if (++q.b >= blk_hi) return false;
        q.s = 0;
        seq_load(p, w, w0_slots, q);
    }
    return true;
}

// One lane: expect the bytes and start the TMA copies of the slot at q.
__device__ __forceinline__ void issue_slot(const DecodeParams &p, const WarpSeq &q, int w0_lo, int w0_hi,
                                           uint8_t *dst, uint64_t *bar) {
    const bool is_u = q.s >= q.nw0;
    const int c_lo = is_u ? q.u_lo + (q.s - q.nw0) * SC : w0_lo + q.s * SC;
    const int c_hi = min(is_u ? q.u_hi : w0_hi, c_lo + SC);
    mbar_arrive_expect_tx(bar, (uint32_t)(c_hi - c_lo) * kDecodeChunkBytes);
    if (!is_u && p.w3d && c_hi - c_lo == SC) {
        tma_load_3d(dst, &p.tm_w3[q.sp], 0, q.row0, c_lo, bar);
    } else {
        const CUtensorMap *tm = is_u ? &p.tm_u[q.sp] : &p.tm_w[q.sp];
        for (int cc = c_lo; cc < c_hi; ++cc)
            tma_load_2d(dst + (cc - c_lo) * kDecodeChunkBytes, tm, cc * CK, q.row0, bar);
    }
}

// acc += U-or-W0 fragment a (16 x 16) times B = T (fp32) split into bf16 high
// and low parts: two MMAs keep fp32-level accuracy for the low-rank product.
__device__ __forceinline__ void mma_split_t(float (&acc)[4], const uint32_t (&a)[4], float t0, float t1,
                                            float t2, float t3) {
    const uint32_t h0 = pack_bf16x2(t0, t1), h1 = pack_bf16x2(t2, t3);
    const uint32_t l0 = pack_bf16x2(t0 - bf16lo(h0), t1 - bf16hi(h0));
    const uint32_t l1 = pack_bf16x2(t2 - bf16lo(h1), t3 - bf16hi(h1));
    mma_bf16(acc, a, h0, h1);
    mma_bf16(acc, a, l0, l1);
}

// One 16 x 64 chunk of W0 (128-byte swizzled in shared memory) times x: the
// four A fragments and all B fragments are loaded before the MMAs.  FULL: all
// 64 columns lie inside K (no tail checks).
template <int NT, bool XS, bool FULL>
__device__ __forceinline__ void w0_chunk(float (&acc)[NT][4], uint32_t cbase, const uint32_t (&swz)[CK / 16],
                                         int kk0, int K, const bool (&nvalid)[NT],
                                         const uint32_t (&xs_lane)[NT],
                                         const __nv_bfloat16 *const (&xg_lane)[NT]) {
    uint32_t a[CK / 16][4];
    uint32_t bx[CK / 16][NT][2];
#pragma unroll
    for (int kq = 0; kq < CK / 16; ++kq) {
        const int kk = kk0 + kq * 16;
        const bool step = FULL || kk < K;
        const bool hi_ok = FULL || kk + 8 < K;
        if (step) ldmatrix_x4(cbase + swz[kq], a[kq]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            uint32_t b0 = 0u, b1 = 0u;
            if (step && nvalid[nt]) {
                if (XS) {
                    b0 = lds32(xs_lane[nt] + (uint32_t)kk * 2u);
                    if (hi_ok) b1 = lds32(xs_lane[nt] + (uint32_t)kk * 2u + 16u);
                } else {
                    b0 = ldg_u32(xg_lane[nt] + kk);
                    if (hi_ok) b1 = ldg_u32(xg_lane[nt] + kk + 8);
                }
            }
            bx[kq][nt][0] = b0;
            bx[kq][nt][1] = b1;
        }
    }
#pragma unroll
    for (int kq = 0; kq < CK / 16; ++kq)
        if (FULL || kk0 + kq * 16 < K)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16(acc[nt], a[kq], bx[kq][nt][0], bx[kq][nt][1]);
}

// One 16 x 64 chunk of U times T (columns j0 .. j0+63 of the rank r).
template <int NT>
__device__ __forceinline__ void u_chunk(float (&acu)[NT][4], uint32_t cbase, const uint32_t (&swz)[CK / 16],
                                        int j0, int r, const float *T, int t_ld, int g, int q,
                                        const bool (&nvalid)[NT]) {
#pragma unroll
    for (int kq = 0; kq < CK / 16; ++kq) {
        const int kk = j0 + kq * 16;
        if (kk >= r) break;
        uint32_t a[4];
        ldmatrix_x4(cbase + swz[kq], a);
        const int j = kk + 2 * q;
        const bool hi_ok = kk + 8 < r;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float t0 = 0.f, t1 = 0.f, t2 = 0.f, t3 = 0.f;
            if (nvalid[nt]) {
                const float *tr = T + (size_t)(nt * 8 + g) * t_ld;
                t0 = tr[j];
                t1 = tr[j + 1];
                if (hi_ok) {
                    t2 = tr[j + 8];
                    t3 = tr[j + 9];
                }
            }
            mma_split_t(acu[nt], a, t0, t1, t2, t3);
        }
    }
}

// out[m * out_ld + j] = sum_{k0 <= k < k1} V[k][j] x[m][k] for j < r and m < M,
// computed by the 256 consumer threads (all must call it) on CUDA cores.  x is
// read from xsrc with row stride xld (shared or global memory).  `red` is
// shared scratch of 256 * 8 floats; each output is a fixed-order sum.
template <int MT>
__device__ void vtx_block(const __nv_bfloat16 *__restrict__ V, int r, int k0, int k1,
                          const __nv_bfloat16 *xsrc, int xld, int M, float *red, float *out,
                          int out_ld) {
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int g8 = r >> 3;
    if (MT <= 8 && (r & 7) == 0 && g8 > 0 && (kDecodeConsumers % g8) == 0) {
        // 16-byte vectors of 8 columns; thread t always sees column group t % g8
        // and every (256 / g8)-th row of the slice.
        const int reps = kDecodeConsumers / g8;
        const int grp = tid % g8, rep = tid / g8;
        float acc[MT][8];
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[m][e] = 0.f;
#pragma unroll 8
        for (int k = k0 + rep; k < k1; k += reps) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(V + (size_t)k * r + grp * 8));
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m < M) {
                    const float xv = __bfloat162float(xsrc[(size_t)m * xld + k]);
                    acc[m][0] = fmaf(bf16lo(v.x), xv, acc[m][0]);
                    acc[m][1] = fmaf(bf16hi(v.x), xv, acc[m][1]);
                    acc[m][2] = fmaf(bf16lo(v.y), xv, acc[m][2]);
                    acc[m][3] = fmaf(bf16hi(v.y), xv, acc[m][3]);
                    acc[m][4] = fmaf(bf16lo(v.z), xv, acc[m][4]);
                    acc[m][5] = fmaf(bf16hi(v.z), xv, acc[m][5]);
                    acc[m][6] = fmaf(bf16lo(v.w), xv, acc[m][6]);
                    acc[m][7] = fmaf(bf16hi(v.w), xv, acc[m][7]);
                }
            }
        }
        // Per token: lanes of a warp sharing a column group (lane % g8) add with
        // a fixed xor tree, then the remaining copies add in order via `red`.
        const bool shuffle = g8 < 32;
        const int nsrc = shuffle ? NW : reps;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            if (m >= M) break;
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = acc[m][e];
            if (shuffle) {
                for (int o = 16; o >= g8; o >>= 1)
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[e] += __shfl_xor_sync(0xffffffffu, v[e], o);
                if (lane < g8)
#pragma unroll
                    for (int e = 0; e < 8; ++e) red[(w * g8 + lane) * 8 + e] = v[e];
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) red[tid * 8 + e] = v[e];
            }
            consumer_sync();
            for (int j = tid; j < r; j += kDecodeConsumers) {
                const int gg = j >> 3, e = j & 7;
                float s = 0.f;
                for (int q = 0; q < nsrc; ++q) s += red[(gg + q * g8) * 8 + e];
                out[(size_t)m * out_ld + j] = s;
            }
            consumer_sync();
        }
    } else if ((r & 1) == 0 && r / 2 <= kDecodeConsumers) {
        // Column pairs (4-byte loads); (256 / pairs) threads split the rows.
        const int P2 = r / 2;
        const int reps = kDecodeConsumers / P2;
        const int pair = tid % P2, rep = tid / P2;
        float acc[MT][2];
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[m][0] = acc[m][1] = 0.f;
        if (rep < reps) {
#pragma unroll 4
            for (int k = k0 + rep; k < k1; k += reps) {
                const uint32_t v = ldg_u32(V + (size_t)k * r + 2 * pair);
                const float v0 = bf16lo(v), v1 = bf16hi(v);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m < M) {
                        const float xv = __bfloat162float(xsrc[(size_t)m * xld + k]);
                        acc[m][0] = fmaf(v0, xv, acc[m][0]);
                        acc[m][1] = fmaf(v1, xv, acc[m][1]);
                    }
                }
            }
        }
        const bool shuffle = (32 % P2) == 0;  // lanes sharing a pair sit in one warp
        const int nsrc = shuffle ? NW : reps;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            if (m >= M) break;
            float v0 = acc[m][0], v1 = acc[m][1];
            if (shuffle) {
                for (int o = 16; o >= P2; o >>= 1) {
                    v0 += __shfl_xor_sync(0xffffffffu, v0, o);
                    v1 += __shfl_xor_sync(0xffffffffu, v1, o);
                }
                if (lane < P2) {
                    red[(w * P2 + lane) * 2 + 0] = v0;
                    red[(w * P2 + lane) * 2 + 1] = v1;
                }
            } else if (rep < reps) {
                red[tid * 2 + 0] = v0;
                red[tid * 2 + 1] = v1;
            }
            consumer_sync();
            for (int j = tid; j < r; j += kDecodeConsumers) {
                const int pj = j >> 1, e = j & 1;
                float s = 0.f;
                for (int q = 0; q < nsrc; ++q) s += red[(pj + q * P2) * 2 + e];
                out[(size_t)m * out_ld + j] = s;
            }
            consumer_sync();
        }
    } else {
        // Odd or very wide ranks: one column per thread per pass.
        for (int jb = 0; jb < r; jb += kDecodeConsumers) {
            const int j = jb + tid;
            if (j < r) {
                float acc[MT];
#pragma unroll
                for (int m = 0; m < MT; ++m) acc[m] = 0.f;
                for (int k = k0; k < k1; ++k) {
                    const float v = __bfloat162float(V[(size_t)k * r + j]);
#pragma unroll
                    for (int m = 0; m < MT; ++m)
                        if (m < M) acc[m] = fmaf(v, __bfloat162float(xsrc[(size_t)m * xld + k]), acc[m]);
                }
                for (int m = 0; m < M; ++m) out[(size_t)m * out_ld + j] = acc[m];
            }
        }
        consumer_sync();
    }
}

struct SmemLayout {
    uint32_t ring_bytes, ts_off, red_off, xs_off, bar_off, flag_off, total;
};

// The ring starts at a 1024-byte boundary (the 128-byte swizzle repeats every
// 1024 bytes); total includes the slack for that alignment.
__host__ __device__ inline SmemLayout smem_layout(int NT, int t_ld, uint32_t x_bytes) {
    const int MT = 8 * NT;
    SmemLayout L;
    L.ring_bytes = (uint32_t)NW * SLOTS * kDecodeSlotBytes;
    L.ts_off = L.ring_bytes;
    L.red_off = L.ts_off + (((uint32_t)(MT * t_ld) * 4u + 127u) & ~127u);
    const uint32_t vtx_red = (uint32_t)kDecodeConsumers * 8u * 4u;
    const uint32_t epi_red = 2u * NW * 32u * 8u * (uint32_t)NT * 4u;
    L.xs_off = L.red_off + (vtx_red > epi_red ? vtx_red : epi_red);
    L.bar_off = L.xs_off + ((x_bytes + 127u) & ~127u);
    L.flag_off = L.bar_off + 2u * NW * SLOTS * 8u;
    L.total = L.flag_off + 16u + 1024u;
    return L;
}

}  // namespace

template <int NT, bool XS>
__global__ void __launch_bounds__(kDecodeThreads, 1)
    decode_kernel(const __grid_constant__ DecodeParams p) {
    constexpr int MT = 8 * NT;
    // The next kernel in the stream may launch now; it waits for this grid
    // before it reads anything this grid writes.
    pdl_launch_dependents();

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    const SmemLayout L = smem_layout(NT, p.t_ld, XS ? (uint32_t)(p.M * p.x_ld * 2) : 0u);
    uint8_t *ring = smem;
    float *Ts = reinterpret_cast<float *>(smem + L.ts_off);    // [M][t_ld]
    float *red = reinterpret_cast<float *>(smem + L.red_off);
    __nv_bfloat16 *xs = reinterpret_cast<__nv_bfloat16 *>(smem + L.xs_off);  // [M][x_ld]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bar_off);  // [NW][SLOTS]
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.flag_off);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int blk_lo = (int)(((long long)blockIdx.x * p.total_blocks) / gridDim.x);
    const int blk_hi = (int)(((long long)(blockIdx.x + 1) * p.total_blocks) / gridDim.x);
    const int K = p.K, M = p.M;

    if (tid == 0) {
        for (int i = 0; i < NW * SLOTS; ++i) mbar_init(&full[i], 1);
        *abort_flag = 0;
        fence_barrier_init();
        for (int i = 0; i < p.nseg; ++i) {
            prefetch_tmap(&p.tm_w[i]);
            if (p.w3d) prefetch_tmap(&p.tm_w3[i]);
            if (p.u_bulk && p.seg[i].r > 0) prefetch_tmap(&p.tm_u[i]);
        }
    }
    __syncthreads();

    // This warp's share of the W0 chunks (the same for every block of the call).
    int w0_lo, w0_hi;
    warp_chunks((K + CK - 1) / CK, warp, w0_lo, w0_hi);
    const int w0_slots = (w0_hi - w0_lo + SC - 1) / SC;

    // Each warp feeds its own SLOTS-deep ring: W0 and U are parameters, so the
    // first copies go out before waiting for the previous kernel.
    uint64_t *my_full = full + warp * SLOTS;
    uint8_t *my_ring = ring + (size_t)warp * SLOTS * kDecodeSlotBytes;
    WarpSeq iq;  // issue position
    iq.b = blk_lo;
    iq.s = -1;
    bool more = blk_lo < blk_hi;
    if (more) {
        seq_load(p, warp, w0_slots, iq);
        iq.s = 0;
        while (iq.s >= iq.ns) {  // blocks where this warp has nothing to stream
            if (++iq.b >= blk_hi) {
                more = false;
                break;
            }
            seq_load(p, warp, w0_slots, iq);
        }
    }
    uint32_t issued = 0;
    for (int i = 0; i < SLOTS && more; ++i) {
        if (lane == 0) issue_slot(p, iq, w0_lo, w0_hi, my_ring + (size_t)i * kDecodeSlotBytes, &my_full[i]);
        ++issued;
        more = seq_next(p, warp, w0_slots, blk_hi, iq);
    }

    pdl_wait_primary();  // the previous kernel is done: x and the scratch are ours
    bool ok = true;
    const __nv_bfloat16 *xsrc = p.x;
    int xld = K;
    if (XS) {
        // x (M x K) into shared memory, rows padded so B-fragment reads are
        // conflict-free; read once from L2 instead of once per row block.
        const int vpr = K / 8;  // 16-byte vectors per row
        for (int i = tid; i < M * vpr; i += kDecodeConsumers) {
            const int m = i / vpr, v = i - m * vpr;
            *reinterpret_cast<uint4 *>(xs + (size_t)m * p.x_ld + v * 8) =
                __ldg(reinterpret_cast<const uint4 *>(p.x + (size_t)m * K + v * 8));
        }
        consumer_sync();
        xsrc = xs;
        xld = p.x_ld;
    }

    // ---- T = V^T x for the projections this CTA's rows belong to ----
    if (p.t_mode == kTLocal) {
        for (int sp = 0; sp < p.nseg; ++sp) {
            const DecodeSeg &sg = p.seg[sp];
            if (seg_touched(sg, blk_lo, blk_hi))
                vtx_block<MT>(sg.V, sg.r, 0, K, xsrc, xld, M, red, Ts + sg.t_off, p.t_ld);
        }
    } else if (p.t_mode == kTGrid) {
        // (1) all partials written -> (2) CTA c adds column block c over all
        // CTAs into Tfin -> (3) every CTA loads the T slices it needs.
        const unsigned grid = gridDim.x;
        const int n_out = M * p.t_ld;
        float *Tfin = p.Tpart + (size_t)grid * n_out;
        const int k_lo = (int)(((long long)blockIdx.x * K) / grid);
        const int k_hi = (int)(((long long)(blockIdx.x + 1) * K) / grid);
        float *part = p.Tpart + (size_t)blockIdx.x * n_out;
        for (int sp = 0; sp < p.nseg; ++sp) {
            const DecodeSeg &sg = p.seg[sp];
            if (sg.r > 0)
                vtx_block<MT>(sg.V, sg.r, k_lo, k_hi, xsrc, xld, M, red, part + sg.t_off, p.t_ld);
        }
        __threadfence();
        consumer_sync();
        bool fail = tid == 0 && !grid_arrive_wait(&p.sync[0], grid, p);
        ok = !consumer_any(fail || *abort_flag != 0);
        if (ok) {
            const int o_lo = (int)(((long long)blockIdx.x * n_out) / grid);
            const int o_hi = (int)(((long long)(blockIdx.x + 1) * n_out) / grid);
            for (int o = o_lo + warp; o < o_hi; o += NW) {
                float s = 0.f;
                for (unsigned c = lane; c < grid; c += 32) s += __ldcg(p.Tpart + (size_t)c * n_out + o);
                s = warp_sum(s);
                if (lane == 0) Tfin[o] = s;
            }
            __threadfence();
            consumer_sync();
            fail = tid == 0 && !grid_arrive_wait(&p.sync[1], grid, p);
            ok = !consumer_any(fail || *abort_flag != 0);
        }
        if (ok) {
            for (int sp = 0; sp < p.nseg; ++sp) {
                const DecodeSeg &sg = p.seg[sp];
                if (!seg_touched(sg, blk_lo, blk_hi)) continue;
                for (int i = tid; i < M * sg.r; i += kDecodeConsumers) {
                    const int m = i / sg.r, j = i - m * sg.r;
                    const size_t o = (size_t)m * p.t_ld + sg.t_off + j;
                    Ts[o] = __ldcg(Tfin + o);
                }
            }
            consumer_sync();
            if (tid == 0) {
                // The last CTA past both arrival counts resets the counters
                // for the next call (nobody polls them any more).
                if (atomicAdd(&p.sync[2], 1u) == grid - 1) {
                    atomicExch(&p.sync[0], 0u);
                    atomicExch(&p.sync[1], 0u);
                    atomicExch(&p.sync[2], 0u);
                }
            }
        }
    }
    ok = !consumer_any(!ok || *abort_flag != 0);

    // ---- row blocks: z = W0 x and U T on the tensor cores ----
    const int g = lane >> 2, q = lane & 3;          // fragment row / column-pair index
    const int lrow = lane & 15, lhalf = lane >> 4;  // ldmatrix source row / k half
    const uint32_t ring_s = smem_addr(my_ring) + (uint32_t)lrow * 128u;
    uint32_t swz[CK / 16];  // ldmatrix offset of k-step kq inside a chunk (128-byte swizzle)
#pragma unroll
    for (int kq = 0; kq < CK / 16; ++kq) swz[kq] = (uint32_t)((kq * 2 + lhalf) ^ (lrow & 7)) << 4;
    // This lane's B-fragment source: x row n = nt*8 + g, column pair 2q.
    bool nvalid[NT];
    uint32_t xs_lane[NT];
    const __nv_bfloat16 *xg_lane[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int n = nt * 8 + g;
        nvalid[nt] = n < M;
        const int nn = nvalid[nt] ? n : 0;
        xs_lane[nt] = smem_addr(xs) + (uint32_t)((nn * p.x_ld + 2 * q) * 2);
        xg_lane[nt] = p.x + (size_t)nn * K + 2 * q;
    }
    uint32_t consumed = 0;
    int buf = 0;
    for (int b = blk_lo; b < blk_hi && ok; ++b) {
        WarpSeq cq;
        cq.b = b;
        cq.s = 0;
        seq_load(p, warp, w0_slots, cq);
        const DecodeSeg &sg = p.seg[cq.sp];
        // The scale of the output this thread writes at the end of the block,
        // fetched now so its latency hides behind the block's MMAs.
        const int n_out = cq.nrows * M;
        const float sc = tid < n_out ? __ldg(sg.s + cq.row0 + tid / M) : 0.f;
        float acc[NT][4], acu[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] = acu[nt][e] = 0.f;

        for (int s = 0; s < cq.ns; ++s) {
            const uint32_t sidx = consumed % SLOTS, ph = (consumed / SLOTS) & 1u;
            if (!warp_wait(&my_full[sidx], ph, p, abort_flag)) {
                ok = false;  // the warps decide together at the block barrier
                break;
            }
            const uint32_t sbase = ring_s + sidx * (uint32_t)kDecodeSlotBytes;
            if (s < cq.nw0) {
                const int c_lo = w0_lo + s * SC;
                const int nch = min(SC, w0_hi - c_lo);
                for (int cc = 0; cc < nch; ++cc) {
                    const uint32_t cbase = sbase + (uint32_t)cc * kDecodeChunkBytes;
                    const int kk0 = (c_lo + cc) * CK;
                    if (kk0 + CK <= K)
                        w0_chunk<NT, XS, true>(acc, cbase, swz, kk0, K, nvalid, xs_lane, xg_lane);
                    else
                        w0_chunk<NT, XS, false>(acc, cbase, swz, kk0, K, nvalid, xs_lane, xg_lane);
                }
            } else {
                const int c_lo = cq.u_lo + (s - cq.nw0) * SC;
                const int nch = min(SC, cq.u_hi - c_lo);
                for (int cc = 0; cc < nch; ++cc)
                    u_chunk<NT>(acu, sbase + (uint32_t)cc * kDecodeChunkBytes, swz, (c_lo + cc) * CK, sg.r,
                                Ts + sg.t_off, p.t_ld, g, q, nvalid);
            }
            ++consumed;
            // Refill this slot with the warp's next copy: every lane's fragments
            // were consumed by the MMAs above; order those generic-proxy reads
            // before the async-proxy write.
            __syncwarp();
            if (more) {
                if (lane == 0) {
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    issue_slot(p, iq, w0_lo, w0_hi, my_ring + (size_t)sidx * kDecodeSlotBytes, &my_full[sidx]);
                }
                ++issued;
                more = seq_next(p, warp, w0_slots, blk_hi, iq);
            }
        }

        // delta without TMA (odd rank or unaligned U): A fragments from global
        if (ok && !p.u_bulk && sg.r > 0) {
            int lo, hi;
            warp_u_chunks(sg.r, warp, lo, hi);
            lo *= CK;
            hi = min(sg.r, hi * CK);
            const float *T = Ts + sg.t_off;
            for (int j0 = lo; j0 < hi; j0 += 16) {
                uint32_t a[4];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const int row = g + 8 * (h & 1), j = j0 + 2 * q + 8 * (h >> 1);
                    float u0 = 0.f, u1 = 0.f;
                    if (row < cq.nrows) {
                        const __nv_bfloat16 *ur = sg.U + (size_t)(cq.row0 + row) * sg.r;
                        if (j < hi) u0 = __bfloat162float(ur[j]);
                        if (j + 1 < hi) u1 = __bfloat162float(ur[j + 1]);
                    }
                    a[h] = pack_bf16x2(u0, u1);
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int j = j0 + 2 * q;
                    float t0 = 0.f, t1 = 0.f, t2 = 0.f, t3 = 0.f;
                    if (nvalid[nt]) {
                        const float *tr = T + (size_t)(nt * 8 + g) * p.t_ld;
                        if (j < hi) t0 = tr[j];
                        if (j + 1 < hi) t1 = tr[j + 1];
                        if (j + 8 < hi) t2 = tr[j + 8];
                        if (j + 9 < hi) t3 = tr[j + 9];
                    }
                    mma_split_t(acu[nt], a, t0, t1, t2, t3);
                }
            }
        }

        // ---- add the eight warps' accumulators; y = s * z + U T ----
        float *rb = red + (size_t)buf * NW * 32 * 8 * NT;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float4 *dst = reinterpret_cast<float4 *>(rb + ((size_t)(warp * 32 + lane) * NT + nt) * 8);
            dst[0] = make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
            dst[1] = make_float4(acu[nt][0], acu[nt][1], acu[nt][2], acu[nt][3]);
        }
        if (consumer_any(!ok || *abort_flag != 0)) {
            ok = false;  // every warp leaves together
            break;
        }
        if (tid < n_out) {  // n_out <= 16 * 16 = the thread count
            const int row = tid / M, n = tid - row * M;
            const int nt = n >> 3, tc = n & 7;
            const int fl = (row & 7) * 4 + (tc >> 1);  // fragment lane
            const int fe = (row >> 3) * 2 + (tc & 1);   // element in that lane
            float z = 0.f, d = 0.f;
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float *f = rb + ((size_t)(w * 32 + fl) * NT + nt) * 8;
                z += f[fe];
                d += f[4 + fe];
            }
            sg.y[(size_t)n * sg.N + cq.row0 + row] = __float2bfloat16_rn(fmaf(sc, z, d));
        }
        buf ^= 1;
    }

    // Copies still in flight (only after an abort) land before the CTA exits.
    for (uint32_t i = consumed; i < issued; ++i)
        mbar_wait(&my_full[i % SLOTS], (i / SLOTS) & 1u, p.status, 1000000ull);
    __syncthreads();
}

// ------------------------------------------------------------------ host ---
wl_status plan_decode(DecodeParams &p, int num_sms, DecodePlan *plan) {
    if (p.M < 1 || p.M > WL_DECODE_MAX_M || p.K < 8 || p.nseg < 1) return WL_ERR_UNSUPPORTED;
    const int NT = (p.M + 7) / 8;
    if ((size_t)8 * NT * p.t_ld > (size_t)kDecodeTMaxFloats) return WL_ERR_UNSUPPORTED;

    int blocks = 0;
    bool any_r = false;
    p.u_bulk = 1;
    for (int i = 0; i < p.nseg; ++i) {
        DecodeSeg &sg = p.seg[i];
        sg.blk_begin = blocks;
        blocks += (sg.N + BR - 1) / BR;
        if (sg.r > 0) {
            any_r = true;
            if (sg.r % 8 != 0 || (reinterpret_cast<uintptr_t>(sg.U) & 15u) != 0) p.u_bulk = 0;
        }
    }
    if (!any_r) p.u_bulk = 0;
    p.total_blocks = blocks;
    p.w3d = (p.K % CK == 0 && p.K / CK >= SC) ? 1 : 0;

    wl_status st;
    for (int i = 0; i < p.nseg; ++i) {
        const DecodeSeg &sg = p.seg[i];
        if ((st = encode_map_2d(&p.tm_w[i], sg.W0, p.K, sg.N, p.K, CK, BR)) != WL_OK) return st;
        if (p.w3d &&
            (st = encode_map_3d(&p.tm_w3[i], sg.W0, CK, sg.N, p.K / CK, (uint64_t)p.K * 2, CK * 2, CK, BR,
                                SC)) != WL_OK)
            return st;
        if (p.u_bulk && sg.r > 0 &&
            (st = encode_map_2d(&p.tm_u[i], sg.U, sg.r, sg.N, sg.r, CK, BR)) != WL_OK)
            return st;
    }

    int grid = blocks < num_sms ? blocks : num_sms;
    if (!any_r) {
        p.t_mode = kTNone;
    } else {
        // local mode when the V bytes any one CTA must read stay small
        size_t worst = 0;
        for (int c = 0; c < grid; ++c) {
            const int lo = (int)(((long long)c * blocks) / grid);
            const int hi = (int)(((long long)(c + 1) * blocks) / grid);
            size_t bytes = 0;
            for (int i = 0; i < p.nseg; ++i) {
                const DecodeSeg &sg = p.seg[i];
                const int nb = (sg.N + BR - 1) / BR;
                if (sg.r > 0 && sg.blk_begin < hi && sg.blk_begin + nb > lo) bytes += (size_t)p.K * sg.r * 2;
            }
            if (bytes > worst) worst = bytes;
        }
        p.t_mode = worst <= kLocalVBytes ? kTLocal : kTGrid;
    }
    // Stage x in shared memory when it fits next to the ring.
    p.x_ld = p.K + 8;
    const uint32_t x_bytes = (uint32_t)p.M * p.x_ld * 2;
    p.x_smem = smem_layout(NT, p.t_ld, x_bytes).total <= kDecodeMaxSmem ? 1 : 0;
    plan->grid = grid;
    plan->smem = smem_layout(NT, p.t_ld, p.x_smem ? x_bytes : 0u).total;
    plan->tpart_bytes = p.t_mode == kTGrid ? (size_t)(grid + 1) * p.M * p.t_ld * sizeof(float) : 0;
    return WL_OK;
}

template <int NT, bool XS>
static cudaError_t launch_decode_nt(const DecodeParams &p, const DecodePlan &plan, cudaStream_t stream) {
    // Opt in to the large shared-memory carve-out once per device.
    static bool attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_done[dev]) {
        e = cudaFuncSetAttribute(decode_kernel<NT, XS>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.grid);
    cfg.blockDim = dim3(kDecodeThreads);
    cfg.dynamicSmemBytes = plan.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_kernel<NT, XS>, p);
}

cudaError_t launch_decode(const DecodeParams &p, const DecodePlan &plan, cudaStream_t stream) {
    if (p.M <= 8)
        return p.x_smem ? launch_decode_nt<1, true>(p, plan, stream) : launch_decode_nt<1, false>(p, plan, stream);
    if (p.M <= 16)
        return p.x_smem ? launch_decode_nt<2, true>(p, plan, stream) : launch_decode_nt<2, false>(p, plan, stream);
    return cudaErrorInvalidValue;
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
