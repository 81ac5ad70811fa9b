// Decode path (M <= 16 tokens): the memory-bound half of the theta-bundle
// linear, y = s (.) (W0 x) + U (V^T x), as ONE kernel per call.
//
// Work split.  The output rows of the (stacked) call are cut into blocks of 16
// rows that never straddle two projections; each CTA (one per SM at most) owns
// a balanced, contiguous range of blocks (in local T mode, below, the CTAs are
// first shared out among the projections so that each CTA needs one V).  For
// every block, each of the eight warps takes a fixed 1/8 share of the
// 64-column chunks of K (and of the rank r), so all warps stream the same
// number of bytes.
//
// Streaming.  Every warp feeds its own ring of shared-memory slots (a slot is
// 16 rows x up to 256 columns, one 3-D TMA box {64, 16, chunks} with 128-byte
// swizzle, or 2-D boxes for a ragged K; no multicast) and refills a slot as
// soon as it has consumed it, so no warp waits for another to free space.
// W0 and U are parameters: the whole ring is requested before the kernel waits
// for the previous kernel in the stream (griddepcontrol.wait), i.e. while that
// kernel still runs.  Calls whose per-CTA share is small use a compact
// variant (at most 110 KB of shared memory, two CTAs per SM), so the next
// call's CTAs become resident beside this call's and stream their W0 during
// its tail.  Rows past the end of a projection are out of bounds for the copy
// and arrive as zeros.
//
// Arithmetic.  Warp-level tensor-core MMAs (m16n8k16, bf16 in, fp32
// accumulate): A = 16 W0 rows read with ldmatrix through the swizzle
// (conflict-free), B = x (token n, column k) from shared memory when it fits,
// else from L1/L2.  U slots go through a second accumulator with B = T split
// into bf16 high and low parts, so the low-rank product keeps fp32-level
// accuracy.  At the end of each step the eight warps' accumulators are added
// in warp order in shared memory and y = s * (W0 x) + U T is rounded once to
// bf16.  The stream is HBM-bound (M flop per byte of W0), so these warp MMAs
// keep the instruction count per byte low without tcgen05's TMEM round trip.
//
// T = V^T x is formed inside the same kernel ("cooperative vtx" of the pages'
// custom op), one of two ways chosen per call on the host:
//  * local: when each CTA's V is small, the CTA reads all of it (bulk-copied
//    into shared memory before the wait when it fits).  Fused (M <= 8, rank
//    <= 32, one projection with a delta per CTA; a variant of its own): the
//    V^T x MMAs run inside the first step's W0 loop on the same x fragments,
//    each warp over its own K chunks, the eight partial sums are added after
//    that step's barrier, and every epilogue adds U T on the CUDA cores from
//    the staged U rows.  Otherwise the CTA forms its T slices before the
//    first block: warp MMAs with A = V^T read by ldmatrix.trans, the warps
//    splitting the k-steps (CUDA cores when V cannot be staged);
//  * grid: otherwise each CTA forms partial sums over a 1/grid slice of K for
//    every projection (the warps splitting the 16-column tiles of r) and
//    writes them to scratch (phase A); then it waits for all CTAs' partials
//    and adds up its 1/grid share of the outputs over all CTAs (phase B);
//    then it waits for all shares and loads the slices it needs (phase C, in
//    step `lag`).  The steps of the three phases depend on the CTA's block
//    count (the chain starts at once for a CTA with few blocks).
//    Meanwhile the W0 stream runs on: in step
//    t a CTA does the W0 part of its block t and the U part of block t - lag,
//    keeping z = W0 x of the blocks in between in shared memory.  The counters
//    reset themselves once every CTA is past both counts.
// Every sum has a fixed order (no float atomics), so results are reproducible.
//
// Prior art: the custom-op kernel on "Quality (Gemma 4 31B)", "Kernel
// optimizations", custom-op path (128-bit loads, warp-shuffle reductions, one
// warp per output row, cooperative V^T x, a single block barrier).  Here the
// W0 stream is staged by TMA, the per-row dot products run on the tensor
// cores, rows are spread evenly over all SMs, and consecutive calls overlap
// through programmatic dependent launch.
#include <atomic>

#include "wl_common.cuh"
#include "wl_internal.h"
#include "wl_prefetch.cuh"

namespace wl {

namespace {

constexpr int NW = kDecodeWarps;
constexpr int NTH = kDecodeThreads;
constexpr int BR = kDecodeBlockRows;
constexpr int CK = kDecodeChunkK;
constexpr size_t kLocalVBytes = 96 * 1024;    // local T when each CTA's V is at most this
constexpr size_t kFusedLocalVBytes = 136 * 1024;  // the same for fused local T and at most two blocks a CTA
constexpr uint32_t kDecodeMaxSmem = 227 * 1024;
constexpr uint32_t kSmallSmem = 110 * 1024;   // two CTAs per SM
constexpr size_t kSmallCtaBytes = 256 * 1024; // W0 + U per CTA up to which a call is small
constexpr uint32_t kMaxRingBytes = 192 * 1024;

__device__ __forceinline__ unsigned int ld_acquire_gpu(const unsigned int *p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_gpu_add(unsigned int *p, unsigned int v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Wait (bounded) until a grid-wide counter reaches `expected`.
__device__ __forceinline__ bool grid_wait(const unsigned int *ctr, unsigned int expected, const DecodeArgs &p) {
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_gpu(ctr) < expected) {
        if (globaltimer_ns() - t0 > p.timeout_ns) {
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

__device__ __forceinline__ Block block_info(const DecodeArgs &p, int b) {
    int sp = 0;
    while (sp + 1 < p.nseg && b >= p.seg[sp + 1].blk_begin) ++sp;
    Block B;
    B.sp = sp;
    B.row0 = (b - p.seg[sp].blk_begin) * BR;
    B.nrows = min(BR, p.seg[sp].N - B.row0);
    return B;
}

__host__ __device__ __forceinline__ int seg_blocks(const DecodeSeg &sg) { return (sg.N + BR - 1) / BR; }

// Blocks [lo, hi) of CTA c out of `grid`: an even split of the whole list, or
// (seg_split) an even split of each projection's blocks over its own CTAs.
__host__ __device__ inline void cta_blocks(const DecodeArgs &p, int c, int grid, int &lo, int &hi) {
    if (!p.seg_split) {
        lo = (int)(((long long)c * p.total_blocks) / grid);
        hi = (int)(((long long)(c + 1) * p.total_blocks) / grid);
        return;
    }
    int sp = 0;
    while (sp + 1 < p.nseg && c >= p.seg[sp + 1].cta_begin) ++sp;
    const DecodeSeg &sg = p.seg[sp];
    const int nc = (sp + 1 < p.nseg ? p.seg[sp + 1].cta_begin : grid) - sg.cta_begin;
    const int nb = seg_blocks(sg), j = c - sg.cta_begin;
    lo = sg.blk_begin + (int)(((long long)j * nb) / nc);
    hi = sg.blk_begin + (int)(((long long)(j + 1) * nb) / nc);
}

__host__ __device__ __forceinline__ bool seg_touched(const DecodeSeg &sg, int blk_lo, int blk_hi) {
    return sg.r > 0 && sg.blk_begin < blk_hi && sg.blk_begin + seg_blocks(sg) > blk_lo;
}

// All lanes wait on the barrier phase; the warp agrees on the outcome.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, const DecodeArgs &p,
                                          volatile int *abort_flag) {
    bool ok = mbar_wait(bar, parity, p.status, p.timeout_ns) && (*abort_flag == 0);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && (threadIdx.x & 31) == 0) *abort_flag = 1;
    return ok;
}

// L2 policy for the streamed operands (W0, U): each byte is read once per
// call, so those lines go first when L2 needs room and the small, reused data
// (x, V, s, T scratch, the kernel's own code and parameters) stays cached.
__device__ __forceinline__ uint64_t stream_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ void tma_stream_2d(void *dst_smem, const void *tmap, int c0, int c1, uint64_t *bar,
                                              uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst_smem)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(smem_addr(bar)), "l"(pol)
        : "memory");
}

__device__ __forceinline__ void tma_stream_3d(void *dst_smem, const void *tmap, int c0, int c1, int c2,
                                              uint64_t *bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_addr(dst_smem)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar)), "l"(pol)
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

// Chunks [lo, hi) of warp w among n chunks.
__host__ __device__ __forceinline__ void warp_chunks(int n, int w, int &lo, int &hi) {
    lo = (w * n) / NW;
    hi = ((w + 1) * n) / NW;
}

// Chunks of the rank r that warp w streams: handed out in reverse warp order,
// so they land first on the warps whose W0 share is one chunk short.
__host__ __device__ __forceinline__ void warp_u_chunks(int r, int w, int &lo, int &hi) {
    warp_chunks((r + CK - 1) / CK, NW - 1 - w, lo, hi);
}

// Blocks [b0, b1) of projection sp among blocks [blk_lo, blk_hi) (empty if none).
__host__ __device__ __forceinline__ void seg_block_range(const DecodeSeg &sg, int blk_lo, int blk_hi, int &b0,
                                                         int &b1) {
    const int nb = (sg.N + kDecodeBlockRows - 1) / kDecodeBlockRows;
    b0 = sg.blk_begin > blk_lo ? sg.blk_begin : blk_lo;
    b1 = sg.blk_begin + nb < blk_hi ? sg.blk_begin + nb : blk_hi;
    if (b1 < b0) b1 = b0;
}

// Staged U (u_stage): the U rows of the CTA's blocks, projection after
// projection, each block a full 16 rows (rows past N are never copied).
// Byte offset of projection sp's rows in that region.
__host__ __device__ inline uint32_t u_stage_off(const DecodeArgs &p, int sp, int blk_lo, int blk_hi) {
    uint32_t off = 0;
    for (int i = 0; i < sp; ++i) {
        if (p.seg[i].r == 0) continue;
        int b0, b1;
        seg_block_range(p.seg[i], blk_lo, blk_hi, b0, b1);
        off += (uint32_t)(b1 - b0) * kDecodeBlockRows * (uint32_t)p.seg[i].r * 2u;
    }
    return off;
}

// A warp's position in its sequence of ring copies.  The CTA's work is a list
// of steps t = 0 .. nblk + lag - 1; step t holds the W0 part of the CTA's
// block t (t < nblk) and then the U part of its block t - lag (t >= lag, when
// that block's projection has a delta).  Every warp walks the same list.
struct WarpSeq {
    int t, part, s;  // step, part (0 = W0, 1 = U), slot within the part
    int ns;          // slots of this part for this warp
    int sp, row0;    // projection and first row of the part's block
    int u_lo, u_hi;  // U chunk range (part 1)
};

__device__ __forceinline__ void seq_load(const DecodeArgs &p, int w, int w0_slots, int blk_lo, int nblk,
                                         WarpSeq &q) {
    q.ns = 0;
    int b;
    if (q.part == 0) {
        if (q.t >= nblk) return;
        b = blk_lo + q.t;
    } else {
        if (q.t < p.lag || q.t - p.lag >= nblk) return;
        b = blk_lo + q.t - p.lag;
    }
    const Block B = block_info(p, b);
    q.sp = B.sp;
    q.row0 = B.row0;
    if (q.part == 0) {
        q.ns = w0_slots;
        return;
    }
    const int r = p.seg[B.sp].r;
    if (!p.u_bulk || p.u_stage || r == 0) return;
    warp_u_chunks(r, w, q.u_lo, q.u_hi);
    q.ns = (q.u_hi - q.u_lo + p.slot_chunks - 1) / p.slot_chunks;
}

// Moves q to the next slot this warp streams; false once the list is done.
__device__ __forceinline__ bool seq_next(const DecodeArgs &p, int w, int w0_slots, int blk_lo, int nblk,
                                         WarpSeq &q) {
    const int nsteps = nblk + p.lag;
    ++q.s;
    while (q.s >= q.ns) {
        if (q.part == 0) {
            q.part = 1;
        } else {
            q.part = 0;
            ++q.t;
        }
        if (q.t >= nsteps) return false;
        q.s = 0;
        seq_load(p, w, w0_slots, blk_lo, nblk, q);
    }
    return true;
}

// Positions q at the first slot of the list; false if it is empty.
__device__ __forceinline__ bool seq_first(const DecodeArgs &p, int w, int w0_slots, int blk_lo, int nblk,
                                          WarpSeq &q) {
    q.t = 0;
    q.part = 0;
    seq_load(p, w, w0_slots, blk_lo, nblk, q);
    q.s = -1;
    return seq_next(p, w, w0_slots, blk_lo, nblk, q);
}

// One lane: expect the bytes and start the TMA copies of the slot at q.
__device__ __forceinline__ void issue_slot(const DecodeParams &P, const DecodeArgs &p, const WarpSeq &q, int w0_lo,
                                           int w0_hi, uint8_t *dst, uint64_t *bar, uint64_t pol) {
    const int sc = p.slot_chunks;
    const bool is_u = q.part == 1;
    const int c_lo = (is_u ? q.u_lo : w0_lo) + q.s * sc;
    const int c_hi = min(is_u ? q.u_hi : w0_hi, c_lo + sc);
    mbar_arrive_expect_tx(bar, (uint32_t)(c_hi - c_lo) * kDecodeChunkBytes);
    if (!is_u && p.w3d && c_hi - c_lo == sc) {
        tma_stream_3d(dst, &P.tm_w3[q.sp], 0, q.row0, c_lo, bar, pol);
    } else {
        const CUtensorMap *tm = is_u ? &P.tm_u[q.sp] : &P.tm_w[q.sp];
        for (int cc = c_lo; cc < c_hi; ++cc)
            tma_stream_2d(dst + (cc - c_lo) * kDecodeChunkBytes, tm, cc * CK, q.row0, bar, pol);
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

// w0_chunk plus, on the same x fragments, the chunk's share of T = V^T x for
// the rank r <= 32 of the CTA's projection (fused local T): A = V^T from the
// staged V rows (row k at k * r) through ldmatrix.trans, rows past K masked.
// A tile's columns past r (FT = 2 with r <= 24, or a projection of rank 16
// in a call whose largest rank needs two tiles) read the following rows'
// values, at most 32 bytes past the staged rows and still inside the CTA's
// shared memory; their sums land in T columns that nothing reads.
template <int NT, int FT, bool FULL>
__device__ __forceinline__ void w0v_chunk(float (&acc)[NT][4], float (&acct)[FT][NT][4], uint32_t cbase,
                                          const uint32_t (&swz)[CK / 16], int kk0, int K,
                                          const bool (&nvalid)[NT], const uint32_t (&xs_lane)[NT],
                                          uint32_t v_lane, int r, int q);

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

// U T for columns [j0, j1) of the rank r (16 at a time) with A = the block's
// 16 staged U rows (row-major, row stride r) read by ldmatrix; urow_lane is
// this lane's row (lane & 15) and column half (lane >> 4) address.  Columns
// past r in a 16-column step are cleared (they would read the next row).
template <int NT>
__device__ __forceinline__ void u_staged(float (&acu)[NT][4], uint32_t urow_lane, int j0, int j1, int r,
                                         const float *T, int t_ld, int g, int q, const bool (&nvalid)[NT]) {
    for (int kk = j0; kk < j1; kk += 16) {
        uint32_t a[4];
        ldmatrix_x4(urow_lane + (uint32_t)kk * 2u, a);
        const bool hi_ok = kk + 8 < r;
        if (!hi_ok) a[2] = a[3] = 0u;
        const int j = kk + 2 * q;
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

// out[m * out_ld + j] = sum_{k0 <= k < k1} V[k][j] x[m][k] for j < r, m < M,
// on the tensor cores (m16n8k16, A = V^T read with ldmatrix.trans from the
// staged rows, B = x, fp32 accumulate): warp w takes the 16-row k-steps
// w, w + 8, ...; the eight warps' partial sums are added in warp order.  Row
// k of V is at vs + (k - k0) * r (16-byte aligned rows, r % 8 == 0); rows
// past k1 may hold anything and are masked.  x is read from xsrc with row
// stride xld (shared memory when XS).  `red` is shared scratch of
// NW * 4 * NT * 128 floats.  All threads must call it; ends with a barrier.
// B fragments of x for the k-step at kb: columns kb + 2q (+1) and kb + 8 + 2q
// (+1) of token rows nt * 8 + g, zero past k1 (k1 is even, so no pair
// straddles it) and for rows past M.
template <int NT, bool XS>
__device__ __forceinline__ void x_frags(uint32_t (&b)[NT][2], const __nv_bfloat16 *xsrc, int xld, int M, int kb,
                                        int k1, int g, int q) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int n = nt * 8 + g;
        b[nt][0] = b[nt][1] = 0u;
        if (n < M) {
            const __nv_bfloat16 *xr = xsrc + (size_t)n * xld + kb + 2 * q;
            if (kb + 2 * q < k1) b[nt][0] = XS ? *reinterpret_cast<const uint32_t *>(xr) : ldg_u32(xr);
            if (kb + 8 + 2 * q < k1) b[nt][1] = XS ? *reinterpret_cast<const uint32_t *>(xr + 8) : ldg_u32(xr + 8);
        }
    }
}

// A fragment of V^T (16 columns j0.. of r x 16 rows kb.. of the staged V)
// through ldmatrix.trans; elements of rows past k1 are cleared.
__device__ __forceinline__ void vt_frag(uint32_t (&a)[4], uint32_t v_lane, int r, int k0, int kb, int k1, int j0,
                                        int q) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                 : "r"(v_lane + (uint32_t)((kb - k0) * r + j0) * 2u));
    if (kb + 16 > k1) {
        if (kb + 2 * q >= k1) a[0] = a[1] = 0u;
        if (kb + 8 + 2 * q >= k1) a[2] = a[3] = 0u;
    }
}

template <int NT, int FT, bool FULL>
__device__ __forceinline__ void w0v_chunk(float (&acc)[NT][4], float (&acct)[FT][NT][4], uint32_t cbase,
                                          const uint32_t (&swz)[CK / 16], int kk0, int K,
                                          const bool (&nvalid)[NT], const uint32_t (&xs_lane)[NT],
                                          uint32_t v_lane, int r, int q) {
    // two k-steps at a time: the fused variant runs under the compact
    // variant's register limit
#pragma unroll
    for (int kh = 0; kh < CK / 32; ++kh) {
        uint32_t a[2][4];
        uint32_t bx[2][NT][2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int kq = kh * 2 + h, kk = kk0 + kq * 16;
            const bool step = FULL || kk < K;
            const bool hi_ok = FULL || kk + 8 < K;
            if (step) ldmatrix_x4(cbase + swz[kq], a[h]);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                uint32_t b0 = 0u, b1 = 0u;
                if (step && nvalid[nt]) {
                    b0 = lds32(xs_lane[nt] + (uint32_t)kk * 2u);
                    if (hi_ok) b1 = lds32(xs_lane[nt] + (uint32_t)kk * 2u + 16u);
                }
                bx[h][nt][0] = b0;
                bx[h][nt][1] = b1;
            }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int kk = kk0 + (kh * 2 + h) * 16;
            if (!(FULL || kk < K)) continue;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16(acc[nt], a[h], bx[h][nt][0], bx[h][nt][1]);
#pragma unroll
            for (int jt = 0; jt < FT; ++jt) {
                uint32_t av[4];
                vt_frag(av, v_lane, r, 0, kk, K, jt * 16, q);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_bf16(acct[jt][nt], av, bx[h][nt][0], bx[h][nt][1]);
            }
        }
    }
}

template <int NT, bool XS>
__device__ void vtx_mma(const __nv_bfloat16 *vs, int r, int k0, int k1, const __nv_bfloat16 *xsrc, int xld,
                        int M, float *red, float *out, int out_ld) {
    constexpr int JT = 4;  // 16-column tiles of r per pass
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int g = lane >> 2, q = lane & 3;
    const int nks = (k1 - k0 + 15) >> 4;
    const int njt = (r + 15) >> 4;
    // ldmatrix.trans source row (k) and column (j) offsets of this lane
    const int lk = (lane & 7) + ((lane >> 4) << 3), lj = ((lane >> 3) & 1) << 3;
    const uint32_t v_lane = smem_addr(vs) + (uint32_t)(lk * r + lj) * 2u;
    if (njt >= NW || nks < NW) {
        // Few k-steps or many column tiles (grid-mode slices): warp w takes
        // the tiles w, w + 8, ... over all k-steps and writes complete sums.
        for (int jt = w; jt < njt; jt += NW) {
            const int j0 = jt * 16;
            float acc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
            for (int ks = 0; ks < nks; ++ks) {
                const int kb = k0 + ks * 16;
                uint32_t b[NT][2], a[4];
                x_frags<NT, XS>(b, xsrc, xld, M, kb, k1, g, q);
                vt_frag(a, v_lane, r, k0, kb, k1, j0, q);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_bf16(acc[nt], a, b[nt][0], b[nt][1]);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int n = nt * 8 + 2 * q, j = j0 + g;
                if (n < M) {
                    if (j < r) out[(size_t)n * out_ld + j] = acc[nt][0];
                    if (j + 8 < r) out[(size_t)n * out_ld + j + 8] = acc[nt][2];
                }
                if (n + 1 < M) {
                    if (j < r) out[(size_t)(n + 1) * out_ld + j] = acc[nt][1];
                    if (j + 8 < r) out[(size_t)(n + 1) * out_ld + j + 8] = acc[nt][3];
                }
            }
        }
        __syncthreads();
        return;
    }
    // Many k-steps, few tiles (local mode): warp w takes the k-steps w, w + 8,
    // ...; the eight warps' partial sums are added in warp order.
    for (int jt0 = 0; jt0 < r; jt0 += 16 * JT) {
        float acc[JT][NT][4];
#pragma unroll
        for (int jt = 0; jt < JT; ++jt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[jt][nt][e] = 0.f;
        for (int ks = w; ks < nks; ks += NW) {
            const int kb = k0 + ks * 16;
            uint32_t b[NT][2];
            x_frags<NT, XS>(b, xsrc, xld, M, kb, k1, g, q);
#pragma unroll
            for (int jt = 0; jt < JT; ++jt) {
                const int j0 = jt0 + jt * 16;
                if (j0 >= r) break;
                uint32_t a[4];
                vt_frag(a, v_lane, r, k0, kb, k1, j0, q);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_bf16(acc[jt][nt], a, b[nt][0], b[nt][1]);
            }
        }
        // partial sums of this pass: red[((w * JT + jt) * NT + nt) * 128 + lane * 4 + e]
#pragma unroll
        for (int jt = 0; jt < JT; ++jt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                *reinterpret_cast<float4 *>(red + ((size_t)(w * JT + jt) * NT + nt) * 128 + lane * 4) =
                    make_float4(acc[jt][nt][0], acc[jt][nt][1], acc[jt][nt][2], acc[jt][nt][3]);
        __syncthreads();
        const int ncol = min(16 * JT, r - jt0);
        for (int i = threadIdx.x; i < M * ncol; i += NTH) {
            const int m = i / ncol, jj = i - m * ncol;
            const int jt = jj >> 4, jr = jj & 15;
            const int nt = m >> 3, col = m & 7;
            const int fl = (jr & 7) * 4 + (col >> 1), fe = (jr >> 3) * 2 + (col & 1);
            float s = 0.f;
            for (int ww = 0; ww < NW; ++ww) s += red[((size_t)(ww * JT + jt) * NT + nt) * 128 + fl * 4 + fe];
            out[(size_t)m * out_ld + jt0 + jj] = s;
        }
        __syncthreads();
    }
}

// The same sum on CUDA cores, for V rows that are not staged (unaligned, odd
// rank, or no room): V row k at V + (k - vk0) * r (global or shared), element
// loads.  Token by token; the threads sharing a column split the rows and add
// their partial sums in thread order through `red` (NTH floats).  All threads
// must call it; ends with a barrier.
__device__ __noinline__ void vtx_cores(const __nv_bfloat16 *V, int vk0, int r, int k0, int k1,
                                       const __nv_bfloat16 *xsrc, int xld, int M, float *red, float *out,
                                       int out_ld) {
    const int tid = threadIdx.x;
    const int cols = r < NTH ? r : NTH;
    const int parts = NTH / cols;
    const int jl = tid % cols, part = tid / cols;
    for (int m = 0; m < M; ++m) {
        for (int jb = 0; jb < r; jb += cols) {
            const int j = jb + jl;
            float s = 0.f;
            if (part < parts && j < r)
                for (int k = k0 + part; k < k1; k += parts)
                    s = fmaf(__bfloat162float(V[(size_t)(k - vk0) * r + j]),
                             __bfloat162float(xsrc[(size_t)m * xld + k]), s);
            red[tid] = s;
            __syncthreads();
            if (tid < cols && jb + tid < r) {
                float t = 0.f;
                for (int pp = 0; pp < parts; ++pp) t += red[pp * cols + tid];
                out[(size_t)m * out_ld + jb + tid] = t;
            }
            __syncthreads();
        }
    }
}

// V rows [k0, k1) of projection sp that CTA c reads to form T (empty if none):
// all of K for the projections its rows touch (local mode), or its 1/grid
// share of the 16-row k-steps of K for every projection with a delta (grid
// mode).
__host__ __device__ inline void v_range(const DecodeArgs &p, int sp, int c, int grid, int blk_lo, int blk_hi,
                                        int &k0, int &k1) {
    const DecodeSeg &sg = p.seg[sp];
    k0 = k1 = 0;
    if (sg.r == 0) return;
    if (p.t_mode == kTLocal) {
        if (seg_touched(sg, blk_lo, blk_hi)) k1 = p.K;
    } else if (p.t_mode == kTGrid) {
        // whole 16-row k-steps, so slice edges never split a column pair
        const int nks = (p.K + 15) / 16;
        k0 = 16 * (int)(((long long)c * nks) / grid);
        k1 = 16 * (int)(((long long)(c + 1) * nks) / grid);
        k0 = k0 < p.K ? k0 : p.K;
        k1 = k1 < p.K ? k1 : p.K;
    }
}

// Local mode: T slices of the projections this CTA's rows touch into Ts.
template <int NT, bool XS>
__device__ void form_t_local(const DecodeArgs &p, int blk_lo, int blk_hi, const __nv_bfloat16 *xsrc, int xld,
                             const uint8_t *vs, float *red, float *Ts) {
    uint32_t off = 0;
    for (int sp = 0; sp < p.nseg; ++sp) {
        const DecodeSeg &sg = p.seg[sp];
        if (!seg_touched(sg, blk_lo, blk_hi)) continue;
        if (p.v_stage)
            vtx_mma<NT, XS>(reinterpret_cast<const __nv_bfloat16 *>(vs + off), sg.r, 0, p.K, xsrc, xld, p.M, red,
                            Ts + sg.t_off, p.t_ld);
        else
            vtx_cores(sg.V, 0, sg.r, 0, p.K, xsrc, xld, p.M, red, Ts + sg.t_off, p.t_ld);
        off += (uint32_t)p.K * (uint32_t)sg.r * 2u;
    }
}

// Grid mode, phase A: partial sums over this CTA's K slice for every
// projection with a delta (zeros for an empty slice: all partials are added),
// then arrive on the first counter.
template <int NT, bool XS>
__device__ void grid_t_partials(const DecodeArgs &p, int blk_lo, int blk_hi, const __nv_bfloat16 *xsrc,
                                int xld, const uint8_t *vs, float *red) {
    const int n_out = p.M * p.t_ld;
    uint32_t off = 0;
    for (int sp = 0; sp < p.nseg; ++sp) {
        const DecodeSeg &sg = p.seg[sp];
        if (sg.r == 0) continue;
        int k0, k1;
        v_range(p, sp, blockIdx.x, gridDim.x, blk_lo, blk_hi, k0, k1);
        float *out = p.Tpart + (size_t)blockIdx.x * n_out + sg.t_off;
        if (p.v_stage)
            vtx_mma<NT, XS>(reinterpret_cast<const __nv_bfloat16 *>(vs + off), sg.r, k0, k1, xsrc, xld, p.M, red,
                            out, p.t_ld);
        else
            vtx_cores(sg.V, 0, sg.r, k0, k1, xsrc, xld, p.M, red, out, p.t_ld);
        off += (uint32_t)(k1 - k0) * (uint32_t)sg.r * 2u;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) red_release_gpu_add(&p.sync[0], 1u);
}

// Grid mode, phase B: once every CTA's partials are in, add up this CTA's
// 1/grid share of the outputs over all CTAs (lanes stride the CTAs, then a
// fixed xor tree; four outputs per warp at a time) into the final T, then
// arrive on the second counter.  Returns the CTA's common verdict.
__device__ bool grid_t_reduce(const DecodeArgs &p, volatile int *abort_flag) {
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const unsigned grid = gridDim.x;
    bool fail = tid == 0 && !grid_wait(&p.sync[0], grid, p);
    if (__syncthreads_or(fail || *abort_flag != 0)) return false;
    const int n_out = p.M * p.t_ld;
    float *Tfin = p.Tpart + (size_t)grid * n_out;
    const int o_lo = (int)(((long long)blockIdx.x * n_out) / grid);
    const int o_hi = (int)(((long long)(blockIdx.x + 1) * n_out) / grid);
    for (int o0 = o_lo + 4 * w; o0 < o_hi; o0 += 4 * NW) {
        float s[4] = {0.f, 0.f, 0.f, 0.f};
        for (unsigned c = lane; c < grid; c += 32) {
            const float *src = p.Tpart + (size_t)c * n_out + o0;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (o0 + i < o_hi) s[i] += __ldcg(src + i);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) s[i] = warp_sum(s[i]);
        if (lane == 0)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (o0 + i < o_hi) Tfin[o0 + i] = s[i];
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) red_release_gpu_add(&p.sync[1], 1u);
    return true;
}

// Grid mode, phase C: once every share is in, load the T slices this CTA's
// rows need into Ts.  The last CTA past both counts resets the counters for
// the next call (nobody polls them any more).
__device__ bool grid_t_load(const DecodeArgs &p, int blk_lo, int blk_hi, float *Ts, volatile int *abort_flag) {
    const int tid = threadIdx.x;
    const unsigned grid = gridDim.x;
    bool fail = tid == 0 && !grid_wait(&p.sync[1], grid, p);
    if (__syncthreads_or(fail || *abort_flag != 0)) return false;
    const float *Tfin = p.Tpart + (size_t)grid * p.M * p.t_ld;
    for (int sp = 0; sp < p.nseg; ++sp) {
        const DecodeSeg &sg = p.seg[sp];
        if (!seg_touched(sg, blk_lo, blk_hi)) continue;
        for (int i = tid; i < p.M * sg.r; i += NTH) {
            const int m = i / sg.r, j = i - m * sg.r;
            const size_t o = (size_t)m * p.t_ld + sg.t_off + j;
            Ts[o] = __ldcg(Tfin + o);
        }
    }
    __syncthreads();
    if (tid == 0 && atomicAdd(&p.sync[2], 1u) == grid - 1) {
        atomicExch(&p.sync[0], 0u);
        atomicExch(&p.sync[1], 0u);
        atomicExch(&p.sync[2], 0u);
    }
    return true;
}

constexpr uint32_t kArgsBytes = (uint32_t)((sizeof(DecodeArgs) + 15) & ~size_t(15));

struct SmemLayout {
    uint32_t slot_bytes, ring_bytes, ts_off, red_off, xs_off, vs_off, us_off, zs_off, bar_off, flag_off, total;
};

// Shared memory opens with the copy of the arguments; the ring starts at the
// next 1024-byte boundary (the 128-byte swizzle repeats every 1024 bytes) and
// the offsets below are relative to it; total includes the slack for that
// alignment.
__host__ __device__ inline SmemLayout smem_layout(const DecodeArgs &p, int NT) {
    SmemLayout L;
    L.slot_bytes = (uint32_t)p.slot_chunks * kDecodeChunkBytes;
    L.ring_bytes = (uint32_t)NW * p.slots * L.slot_bytes;
    L.ts_off = L.ring_bytes;
    L.red_off = L.ts_off + (((uint32_t)(p.M * p.t_ld) * 4u + 127u) & ~127u);
    const uint32_t epi_red = 2u * NW * 32u * 8u * (uint32_t)NT * 4u;  // two step buffers
    const uint32_t vtx_red = (uint32_t)NW * 4u * (uint32_t)NT * 128u * 4u;
    L.xs_off = L.red_off + (epi_red > vtx_red ? epi_red : vtx_red);
    const uint32_t x_bytes = p.x_smem ? (uint32_t)p.M * p.x_ld * 2u : 0u;
    L.vs_off = L.xs_off + ((x_bytes + 127u) & ~127u);
    const uint32_t v_bytes = (p.v_stage && !p.v_in_ring) ? (uint32_t)p.v_bytes : 0u;
    L.zs_off = L.vs_off + ((v_bytes + 127u) & ~127u);
    const uint32_t u_bytes = p.u_stage ? (uint32_t)p.u_bytes : 0u;
    L.us_off = L.zs_off;
    L.zs_off = L.us_off + ((u_bytes + 127u) & ~127u);
    const uint32_t z_bytes = p.lag > 0 ? (uint32_t)(p.lag + 1) * BR * p.M * 4u : 0u;
    L.bar_off = L.zs_off + ((z_bytes + 127u) & ~127u);
    L.flag_off = L.bar_off + (uint32_t)(NW * p.slots + 6) * 8u;
    L.total = L.flag_off + 16u + 1024u + kArgsBytes;  // + the copy of the arguments, before the ring
    return L;
}

// What step t of a CTA holds (see WarpSeq).
struct Step {
    bool has_w, has_u;  // W0 part of block t / U part of block t - lag exist
    Block bw, bu;
    int rw, ru;         // ranks of those blocks' projections
};

__device__ __forceinline__ Step step_info(const DecodeArgs &p, int blk_lo, int nblk, int t) {
    Step S;
    S.has_w = t < nblk;
    S.has_u = t >= p.lag && t - p.lag < nblk;
    S.bw = S.has_w ? block_info(p, blk_lo + t) : Block{0, 0, 0};
    S.bu = S.has_u ? block_info(p, blk_lo + t - p.lag) : Block{0, 0, 0};
    S.rw = S.has_w ? p.seg[S.bw.sp].r : 0;
    S.ru = S.has_u ? p.seg[S.bu.sp].r : 0;
    return S;
}

// The scales for output index o of step t's epilogue: for y of block t
// (written then when it has no delta or lag is 0) and of block t - lag.
__device__ __forceinline__ void step_scales(const DecodeArgs &p, const Step &S, int o, float &sc_w,
                                            float &sc_u) {
    const int M = p.M;
    sc_w = sc_u = 0.f;
    if (o < 0) return;
    if (S.has_w && (S.rw == 0 || p.lag == 0) && o < S.bw.nrows * M)
        sc_w = __ldg(p.seg[S.bw.sp].s + S.bw.row0 + o / M);
    if (S.has_u && S.ru > 0 && p.lag > 0 && o < S.bu.nrows * M)
        sc_u = __ldg(p.seg[S.bu.sp].s + S.bu.row0 + o / M);
}

}  // namespace

template <int NT, bool XS, bool SMALL, int FT>
__global__ void __launch_bounds__(NTH, SMALL ? 2 : 1) decode_kernel(const __grid_constant__ DecodeParams P) {
    // The next kernel in the stream may launch now; it waits for this grid
    // before it reads anything this grid writes.
    pdl_launch_dependents();

    // All threads copy the arguments into shared memory (one round of
    // parallel loads); everything below reads that copy.
    extern __shared__ __align__(16) uint8_t smem_raw[];
    {
        const uint32_t *src = reinterpret_cast<const uint32_t *>(&P.a);
        uint32_t *dst = reinterpret_cast<uint32_t *>(smem_raw);
        for (int i = threadIdx.x; i < (int)(sizeof(DecodeArgs) / 4); i += NTH) dst[i] = src[i];
    }
    __syncthreads();
    const DecodeArgs &p = *reinterpret_cast<const DecodeArgs *>(smem_raw);
    int blk_lo, blk_hi;
    cta_blocks(p, blockIdx.x, gridDim.x, blk_lo, blk_hi);
    const int nblk = blk_hi - blk_lo;
    // Grid-mode T schedule of this CTA: phase A (partial sums) in step t_a,
    // phase B (the reduction) in step t_b, phase C (T loaded) in step lag,
    // which is where the first U part runs.  With few blocks there is little
    // W0 to overlap, so the chain starts at once; with many, phase A waits
    // for the first step's W0 part (the stream is under way) unless V holds
    // a ring level, whose copies stop until phase A is done.
    int t_a = 0, t_b = 0;
    if (p.t_mode == kTGrid) {
        int lag;
        if (nblk <= 1) {
            lag = 1;
        } else if (nblk <= 3 || p.v_in_ring) {
            t_b = 1;
            lag = 2;
        } else {
            t_a = 1;
            t_b = 2;
            lag = 3;
        }
        __syncthreads();  // every thread has read the copied arguments
        if (threadIdx.x == 0) reinterpret_cast<DecodeArgs *>(smem_raw)->lag = lag;
        __syncthreads();
    }
    const uint32_t raw_addr = smem_addr(smem_raw) + kArgsBytes;
    uint8_t *smem = smem_raw + kArgsBytes + ((1024u - (raw_addr & 1023u)) & 1023u);
    const SmemLayout L = smem_layout(p, NT);
    uint8_t *ring = smem;
    float *Ts = reinterpret_cast<float *>(smem + L.ts_off);    // [M][t_ld]
    float *red = reinterpret_cast<float *>(smem + L.red_off);  // step sums; T scratch before the steps
    __nv_bfloat16 *xs = reinterpret_cast<__nv_bfloat16 *>(smem + L.xs_off);  // [M][x_ld]
    float *zs = reinterpret_cast<float *>(smem + L.zs_off);    // [lag + 1][16 * M]: z awaiting U T
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bar_off);  // [NW][slots]
    const int SLOTS = p.slots;
    uint64_t *vbar = full + NW * SLOTS;  // V rows staged
    uint64_t *red_full = vbar + 1;       // [2] every warp's sums of a step are in
    uint64_t *red_empty = vbar + 3;      // [2] the step's epilogue has read them
    uint64_t *ubar = vbar + 5;           // U rows staged
    const uint8_t *us = smem + L.us_off;  // staged U rows (u_stage)
    // staged V rows: their own region, or the ring's last slot level (handed
    // to the W0 stream once T's sums are formed)
    uint8_t *vs = p.v_in_ring ? smem + (size_t)(SLOTS - 1) * NW * L.slot_bytes : smem + L.vs_off;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.flag_off);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int nsteps = nblk + p.lag;
    const int K = p.K, M = p.M, SC = p.slot_chunks;

    if (tid == 0) {
        for (int i = 0; i < NW * SLOTS + 1; ++i) mbar_init(&full[i], 1);
        mbar_init(ubar, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&red_full[i], NW);
            mbar_init(&red_empty[i], (BR * p.M + 31) / 32);
        }
        *abort_flag = 0;
        fence_barrier_init();
        for (int i = 0; i < p.nseg; ++i) {
            prefetch_tmap(&P.tm_w[i]);
            if (p.w3d) prefetch_tmap(&P.tm_w3[i]);
            if (p.u_bulk && p.seg[i].r > 0) prefetch_tmap(&P.tm_u[i]);
        }
    }
    __syncthreads();

    // This warp's share of the W0 chunks (the same for every block of the call).
    int w0_lo, w0_hi;
    warp_chunks((K + CK - 1) / CK, warp, w0_lo, w0_hi);
    const int w0_slots = (w0_hi - w0_lo + SC - 1) / SC;

    // Each warp feeds its own ring; W0, U, V and s are parameters, so the V
    // rows for T and the whole ring are requested before waiting for the
    // previous kernel.
    // Slot s of warp w is at ring + (s * NW + w) * slot_bytes (slot-major, so
    // one slot level is contiguous).
    uint64_t *my_full = full + warp * SLOTS;
    uint8_t *my_ring = ring + (size_t)warp * L.slot_bytes;
    const uint32_t level_bytes = (uint32_t)NW * L.slot_bytes;
    const uint64_t pol = stream_policy();
    WarpSeq iq;  // issue position
    bool more = seq_first(p, warp, w0_slots, blk_lo, nblk, iq);
    uint32_t issued = 0;
    int isl = 0;  // ring slot of the next copy
    auto issue_next = [&]() {
        if (lane == 0)
            issue_slot(P, p, iq, w0_lo, w0_hi, my_ring + (size_t)isl * level_bytes, &my_full[isl], pol);
        ++issued;
        if (++isl == SLOTS) isl = 0;
        more = seq_next(p, warp, w0_slots, blk_lo, nblk, iq);
    };
    if (p.v_stage && tid == 0) {
        uint32_t total = 0;
        for (int sp = 0; sp < p.nseg; ++sp) {
            int k0, k1;
            v_range(p, sp, blockIdx.x, gridDim.x, blk_lo, blk_hi, k0, k1);
            total += (uint32_t)(k1 - k0) * (uint32_t)p.seg[sp].r * 2u;
        }
        mbar_arrive_expect_tx(vbar, total);
        uint32_t off = 0;
        for (int sp = 0; sp < p.nseg; ++sp) {
            int k0, k1;
            v_range(p, sp, blockIdx.x, gridDim.x, blk_lo, blk_hi, k0, k1);
            const uint32_t bytes = (uint32_t)(k1 - k0) * (uint32_t)p.seg[sp].r * 2u;
            if (bytes) bulk_load(vs + off, p.seg[sp].V + (size_t)k0 * p.seg[sp].r, bytes, vbar);
            off += bytes;
        }
    }
    if (p.u_stage && tid == 32) {
        // the U rows of this CTA's blocks (full 16-row blocks in shared memory;
        // only rows below N are copied)
        uint32_t total = 0;
        for (int sp = 0; sp < p.nseg; ++sp) {
            const DecodeSeg &sg = p.seg[sp];
            if (sg.r == 0) continue;
            int b0, b1;
            seg_block_range(sg, blk_lo, blk_hi, b0, b1);
            const int r0 = (b0 - sg.blk_begin) * BR, r1 = min(sg.N, (b1 - sg.blk_begin) * BR);
            if (r1 > r0) total += (uint32_t)(r1 - r0) * (uint32_t)sg.r * 2u;
        }
        mbar_arrive_expect_tx(ubar, total);
        for (int sp = 0; sp < p.nseg; ++sp) {
            const DecodeSeg &sg = p.seg[sp];
            if (sg.r == 0) continue;
            int b0, b1;
            seg_block_range(sg, blk_lo, blk_hi, b0, b1);
            const int r0 = (b0 - sg.blk_begin) * BR, r1 = min(sg.N, (b1 - sg.blk_begin) * BR);
            if (r1 > r0)
                bulk_load(const_cast<uint8_t *>(us) + u_stage_off(p, sp, blk_lo, blk_hi),
                          sg.U + (size_t)r0 * sg.r, (uint32_t)(r1 - r0) * (uint32_t)sg.r * 2u, ubar);
        }
    }
    // the whole ring, less the level that holds V until T's sums are formed
    const uint32_t pre_slots = p.v_in_ring ? (uint32_t)SLOTS - 1u : (uint32_t)SLOTS;
    while (more && issued < pre_slots) issue_next();
    // the following call's weights into L2, behind this CTA's own copies
    if (tid == NTH - 32) l2_prefetch_share(P.pf, blockIdx.x, gridDim.x);
    // Output index of this thread in the epilogue of step u (-1: not its turn).
    const int E = (BR * M + 31) / 32;  // warps per epilogue
    auto epi_out = [&](int u) -> int {
        const int rel = (warp - (u * E) % NW + NW) % NW;
        return rel < E ? rel * 32 + lane : -1;
    };
    Step S = step_info(p, blk_lo, nblk, 0);
    float sc_w, sc_u;
    step_scales(p, S, epi_out(0), sc_w, sc_u);

    pdl_wait_primary();  // the previous kernel is done: x and the scratch are ours
    const __nv_bfloat16 *xsrc = p.x;
    int xld = K;
    if (XS) {
        // x (M x K) into shared memory, rows padded so B-fragment reads are
        // conflict-free; read once from L2 instead of once per block.
        const int vpr = K / 8;  // 16-byte vectors per row
        for (int i = tid; i < M * vpr; i += NTH) {
            const int m = i / vpr, v = i - m * vpr;
            *reinterpret_cast<uint4 *>(xs + (size_t)m * p.x_ld + v * 8) =
                __ldg(reinterpret_cast<const uint4 *>(p.x + (size_t)m * K + v * 8));
        }
        __syncthreads();
        xsrc = xs;
        xld = p.x_ld;
    }

    bool ok = true;
    if (p.t_mode != kTNone && p.v_stage)
        ok = !__syncthreads_or(!mbar_wait(vbar, 0, p.status, p.timeout_ns) || *abort_flag != 0);
    // Fused local T (FT > 0: a variant of its own, launched for t_fused with
    // FT 16-column tiles of the rank): the one projection with a delta that
    // this CTA's rows touch; its V rows open the staged region.
    constexpr bool fused = FT > 0;
    int t_sp = -1;
    if (fused)
        for (int sp = 0; sp < p.nseg && t_sp < 0; ++sp)
            if (seg_touched(p.seg[sp], blk_lo, blk_hi)) t_sp = sp;
    // fused: the epilogues read the staged U rows from the first step on
    if (ok && fused && p.u_stage)
        ok = !__syncthreads_or(!mbar_wait(ubar, 0, p.status, p.timeout_ns) || *abort_flag != 0);
    if (ok && p.t_mode == kTLocal && !fused) form_t_local<NT, XS>(p, blk_lo, blk_hi, xsrc, xld, vs, red, Ts);


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
    // Fused local T: the warp's partial sums over its K chunks.
    constexpr int FTA = FT > 0 ? FT : 1;
    float acct[FTA][NT][4];
#pragma unroll
    for (int jt = 0; jt < FTA; ++jt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acct[jt][nt][e] = 0.f;

    bool u_ready = false;  // the staged U rows have been waited for
    uint32_t consumed = 0;
    int csl = 0;       // ring slot of the next copy to consume
    uint32_t cph = 0;  // its barrier phase parity
    // While the ring's last level holds V, the copies (which take the slots in
    // rotation) stop before it.
    bool v_held = p.v_in_ring != 0;
    // Consumed the slot: every lane's fragments were used by the MMAs above;
    // order those generic-proxy reads before the async-proxy refill.
    auto release_slot = [&]() {
        ++consumed;
        if (++csl == SLOTS) {
            csl = 0;
            cph ^= 1u;
        }
        __syncwarp();
        if (more && !v_held) {
            if (lane == 0) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue_next();
        }
    };
    // Once every thread is past its reads of V (the T routines end with a
    // barrier), the level that held V goes back to the W0 stream and the ring
    // is topped up.
    auto release_v_level = [&]() {
        v_held = false;
        if (lane == 0) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        while (more && issued < consumed + (uint32_t)SLOTS) issue_next();
    };
    if (p.v_in_ring && p.t_mode == kTLocal) release_v_level();

    // Epilogue of step u: the warp's share of y for the blocks of step u (or
    // z kept for a later U part), from all warps' sums in buffer u & 1.  It
    // is done by E consecutive warps starting at (u * E) % NW, so the work
    // rotates over the warps; wait_full: wait for all warps' sums first.
    auto epilogue = [&](int u, const Step &Su, float su_w, float su_u, bool wait_full) -> bool {
        const int o = epi_out(u);
        if (o < 0) return true;
        const int b = u & 1;
        if (wait_full && !warp_wait(&red_full[b], (uint32_t)(u >> 1) & 1u, p, abort_flag)) return false;
        const float *rbu = red + (size_t)b * NW * 32 * 8 * NT;
        if (o < BR * M) {
            const int row = o / M, n = o - row * M;
            const int nt = n >> 3, tc = n & 7;
            const int fl = (row & 7) * 4 + (tc >> 1);  // fragment lane
            const int fe = (row >> 3) * 2 + (tc & 1);   // element in that lane
            float z = 0.f, d = 0.f;
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float *f = rbu + ((size_t)(w * 32 + fl) * NT + nt) * 8;
                z += f[fe];
                d += f[4 + fe];
            }
            if (fused && Su.has_w && Su.rw > 0 && row < Su.bw.nrows) {
                // U T of this output: the staged U row times token n's T slice
                const DecodeSeg &sg = p.seg[Su.bw.sp];
                int b0, b1;
                seg_block_range(sg, blk_lo, blk_hi, b0, b1);
                const __nv_bfloat16 *ur = reinterpret_cast<const __nv_bfloat16 *>(
                                              us + u_stage_off(p, Su.bw.sp, blk_lo, blk_hi)) +
                                          (size_t)(Su.bw.row0 - (b0 - sg.blk_begin) * BR + row) * Su.rw;
                const float *tr = Ts + (size_t)n * p.t_ld + sg.t_off;
                d = 0.f;
                for (int j = 0; j < Su.rw; j += 8) {
                    const uint4 uv = *reinterpret_cast<const uint4 *>(ur + j);
                    const float4 ta = *reinterpret_cast<const float4 *>(tr + j);
                    const float4 tb = *reinterpret_cast<const float4 *>(tr + j + 4);
                    d = fmaf(bf16lo(uv.x), ta.x, d);
                    d = fmaf(bf16hi(uv.x), ta.y, d);
                    d = fmaf(bf16lo(uv.y), ta.z, d);
                    d = fmaf(bf16hi(uv.y), ta.w, d);
                    d = fmaf(bf16lo(uv.z), tb.x, d);
                    d = fmaf(bf16hi(uv.z), tb.y, d);
                    d = fmaf(bf16lo(uv.w), tb.z, d);
                    d = fmaf(bf16hi(uv.w), tb.w, d);
                }
            }
            if (Su.has_w && row < Su.bw.nrows) {
                const DecodeSeg &sg = p.seg[Su.bw.sp];
                if (Su.rw > 0 && p.lag > 0)
                    zs[(u % (p.lag + 1)) * BR * M + o] = z;  // y once U T of the block is in
                else
                    sg.y[(size_t)n * sg.N + Su.bw.row0 + row] =
                        __float2bfloat16_rn(fmaf(su_w, z, p.lag == 0 ? d : 0.f));
            }
            if (Su.has_u && Su.ru > 0 && p.lag > 0 && row < Su.bu.nrows) {
                const DecodeSeg &sg = p.seg[Su.bu.sp];
                const float zu = zs[((u - p.lag) % (p.lag + 1)) * BR * M + o];
                sg.y[(size_t)n * sg.N + Su.bu.row0 + row] = __float2bfloat16_rn(fmaf(su_u, zu, d));
            }
        }
        if (!SMALL) {  // the compact variant's steps all end with a CTA barrier
            __syncwarp();
            if (lane == 0) mbar_arrive(&red_empty[b]);
        }
        return true;
    };
    int pend = -1;  // step whose epilogue is still due
    float scp_w = 0.f, scp_u = 0.f;
    for (int t = 0; t < nsteps && ok; ++t) {
        if (p.t_mode == kTGrid) {
            if (t == t_a) {
                grid_t_partials<NT, XS>(p, blk_lo, blk_hi, xsrc, xld, vs, red);
                if (p.v_in_ring) release_v_level();
            }
            if (t == t_b) ok = grid_t_reduce(p, abort_flag);
            if (ok && t == p.lag) ok = grid_t_load(p, blk_lo, blk_hi, Ts, abort_flag);
            if (!ok) break;
        }
        float acc[NT][4], acu[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] = acu[nt][e] = 0.f;

        // ---- W0 part of block t: z = W0 x ----
        for (int s = 0; S.has_w && s < w0_slots && ok; ++s) {
            if (!warp_wait(&my_full[csl], cph, p, abort_flag)) {
                ok = false;  // the warps decide together at the step barrier
                break;
            }
            const uint32_t sbase = ring_s + (uint32_t)csl * level_bytes;
            const int c_lo = w0_lo + s * SC;
            const int nch = min(SC, w0_hi - c_lo);
            for (int cc = 0; cc < nch; ++cc) {
                const uint32_t cbase = sbase + (uint32_t)cc * kDecodeChunkBytes;
                const int kk0 = (c_lo + cc) * CK;
                if (fused && t == 0 && t_sp >= 0) {
                    const int t_r = p.seg[t_sp].r;
                    const uint32_t tv_lane =
                        smem_addr(vs) +
                        (uint32_t)((((lane & 7) + ((lane >> 4) << 3)) * t_r + (((lane >> 3) & 1) << 3)) * 2);
                    if (kk0 + CK <= K)
                        w0v_chunk<NT, FTA, true>(acc, acct, cbase, swz, kk0, K, nvalid, xs_lane, tv_lane, t_r, q);
                    else
                        w0v_chunk<NT, FTA, false>(acc, acct, cbase, swz, kk0, K, nvalid, xs_lane, tv_lane, t_r, q);
                } else if (kk0 + CK <= K) {
                    w0_chunk<NT, XS, true>(acc, cbase, swz, kk0, K, nvalid, xs_lane, xg_lane);
                } else {
                    w0_chunk<NT, XS, false>(acc, cbase, swz, kk0, K, nvalid, xs_lane, xg_lane);
                }
            }
            release_slot();
        }

        // ---- U part of block t - lag: U T ----
        const bool u_part = S.has_u && S.ru > 0 && !fused;
        const DecodeSeg &sgu = p.seg[S.bu.sp];
        if (u_part && p.u_bulk && !p.u_stage && ok) {
            int u_lo, u_hi;
            warp_u_chunks(S.ru, warp, u_lo, u_hi);
            const int nu = (u_hi - u_lo + SC - 1) / SC;
            for (int s = 0; s < nu; ++s) {
                if (!warp_wait(&my_full[csl], cph, p, abort_flag)) {
                    ok = false;
                    break;
                }
                const uint32_t sbase = ring_s + (uint32_t)csl * level_bytes;
                const int c_lo = u_lo + s * SC;
                const int nch = min(SC, u_hi - c_lo);
                for (int cc = 0; cc < nch; ++cc)
                    u_chunk<NT>(acu, sbase + (uint32_t)cc * kDecodeChunkBytes, swz, (c_lo + cc) * CK, S.ru,
                                Ts + sgu.t_off, p.t_ld, g, q, nvalid);
                release_slot();
            }
        }
        if (u_part && p.u_stage && ok) {
            if (!u_ready) {
                ok = warp_wait(ubar, 0, p, abort_flag);
                u_ready = true;
            }
            if (ok) {
                int u_lo, u_hi;
                warp_u_chunks(S.ru, warp, u_lo, u_hi);
                int b0, b1;
                seg_block_range(sgu, blk_lo, blk_hi, b0, b1);
                // this lane's ldmatrix row (lane & 15) and column half of the block
                const uint32_t urow = smem_addr(us) + u_stage_off(p, S.bu.sp, blk_lo, blk_hi) +
                                      (uint32_t)(((S.bu.row0 - (b0 - sgu.blk_begin) * BR) + (lane & 15)) * S.ru +
                                                 (lane >> 4) * 8) * 2u;
                u_staged<NT>(acu, urow, u_lo * CK, min(S.ru, u_hi * CK), S.ru, Ts + sgu.t_off, p.t_ld, g, q,
                             nvalid);
            }
        }
        if (u_part && !p.u_bulk && ok) {
            // delta without TMA (odd rank or unaligned U): A fragments from global
            int lo, hi;
            warp_u_chunks(S.ru, warp, lo, hi);
            lo *= CK;
            hi = min(S.ru, hi * CK);
            const float *T = Ts + sgu.t_off;
            for (int j0 = lo; j0 < hi; j0 += 16) {
                uint32_t a[4];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const int row = g + 8 * (h & 1), j = j0 + 2 * q + 8 * (h >> 1);
                    float u0 = 0.f, u1 = 0.f;
                    if (row < S.bu.nrows) {
                        const __nv_bfloat16 *ur = sgu.U + (size_t)(S.bu.row0 + row) * S.ru;
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

        // fused T: this warp's partial sums go to the second step buffer,
        // which step 1 fills only after T is added up
        if (fused && t == 0 && ok) {
            float *tred = red + (size_t)NW * 32 * 8 * NT;
#pragma unroll
            for (int jt = 0; jt < FTA; ++jt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    *reinterpret_cast<float4 *>(tred + ((size_t)(warp * FTA + jt) * NT + nt) * 128 + lane * 4) =
                        make_float4(acct[jt][nt][0], acct[jt][nt][1], acct[jt][nt][2], acct[jt][nt][3]);
        }
        // ---- publish this warp's sums of step t ----
        const int rbuf = t & 1;
        float *rb = red + (size_t)rbuf * NW * 32 * 8 * NT;
        // the buffer is free once the epilogue of step t - 2 has read it
        if (!SMALL && ok && t >= 2)
            ok = warp_wait(&red_empty[rbuf], (uint32_t)((t - 2) >> 1) & 1u, p, abort_flag);
        if (ok) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float4 *dst = reinterpret_cast<float4 *>(rb + ((size_t)(warp * 32 + lane) * NT + nt) * 8);
                dst[0] = make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
                dst[1] = make_float4(acu[nt][0], acu[nt][1], acu[nt][2], acu[nt][3]);
            }
            if (!SMALL) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&red_full[rbuf]);
            }
        }
        // Steps of a short call, and steps that carry grid-mode T phases (the
        // phases need every warp), end with a CTA barrier and their epilogue;
        // elsewhere no warp waits for the others except through the two
        // buffers, and the epilogue runs one step behind.
        const bool sync_step = SMALL || (p.t_mode == kTGrid && t <= p.lag) || (fused && t == 0);
        if (sync_step) {
            if (__syncthreads_or(!ok || *abort_flag != 0)) {
                ok = false;  // every warp leaves together
                break;
            }
        } else if (!ok) {
            break;
        }
        if (fused && t == 0) {
            // T of the CTA's projection: the eight warps' partial sums, added
            // in warp order (fragment element (j, token m) of tile jt, nt)
            if (t_sp >= 0) {
                const float *tred = red + (size_t)NW * 32 * 8 * NT;
                const int t_off = p.seg[t_sp].t_off, t_r = p.seg[t_sp].r;
                for (int i = tid; i < M * t_r; i += NTH) {
                    const int m = i / t_r, j = i - m * t_r;
                    const int jt = j >> 4, jr = j & 15, nt = m >> 3, col = m & 7;
                    const int fl = (jr & 7) * 4 + (col >> 1), fe = (jr >> 3) * 2 + (col & 1);
                    float sum = 0.f;
                    for (int w = 0; w < NW; ++w) sum += tred[((size_t)(w * FTA + jt) * NT + nt) * 128 + fl * 4 + fe];
                    Ts[(size_t)m * p.t_ld + t_off + j] = sum;
                }
            }
            __syncthreads();
        }
        const Step cur = S;
        const float cur_sc_w = sc_w, cur_sc_u = sc_u;
        if (t + 1 < nsteps) {
            // the next step's blocks and scales, loaded now so their latency
            // hides behind the next step's MMAs
            S = step_info(p, blk_lo, nblk, t + 1);
            step_scales(p, S, epi_out(t + 1), sc_w, sc_u);
        }
        if (sync_step) {
            ok = epilogue(t, cur, cur_sc_w, cur_sc_u, false);
        } else {
            // the epilogue runs one step behind the MMAs
            if (pend >= 0) ok = epilogue(pend, step_info(p, blk_lo, nblk, pend), scp_w, scp_u, true);
            pend = t;
            scp_w = cur_sc_w;
            scp_u = cur_sc_u;
        }
        if (!ok) break;
    }
    if (ok && pend >= 0) ok = epilogue(pend, step_info(p, blk_lo, nblk, pend), scp_w, scp_u, true);

    // Copies still in flight (only after an abort) land before the CTA exits.
    while (consumed < issued) {
        mbar_wait(&my_full[csl], cph, p.status, 1000000ull);
        ++consumed;
        if (++csl == SLOTS) {
            csl = 0;
            cph ^= 1u;
        }
    }
    if (tid == 0 && p.v_stage) mbar_wait(vbar, 0, p.status, 1000000ull);
    if (tid == 32 && p.u_stage) mbar_wait(ubar, 0, p.status, 1000000ull);
}

// ------------------------------------------------------------------ host ---
namespace {

bool aligned_to(const void *ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

// Shares `grid` CTAs out among the projections: one each, then one at a time
// to the projection with the most blocks per CTA (never more CTAs than blocks).
void split_ctas(DecodeArgs &p, int grid) {
    int ncta[kMaxSeg];
    int used = 0;
    for (int i = 0; i < p.nseg; ++i) {
        ncta[i] = 1;
        ++used;
    }
    while (used < grid) {
        int best = -1, best_load = 0;
        for (int i = 0; i < p.nseg; ++i) {
            const int nb = seg_blocks(p.seg[i]);
            if (ncta[i] >= nb) continue;
            const int load = (nb + ncta[i] - 1) / ncta[i];
            if (load > best_load) {
                best_load = load;
                best = i;
            }
        }
        if (best < 0) break;
        ++ncta[best];
        ++used;
    }
    int c = 0;
    for (int i = 0; i < p.nseg; ++i) {
        p.seg[i].cta_begin = c;
        c += ncta[i];
    }
}

}  // namespace

wl_status plan_decode(DecodeParams &p, int num_sms, DecodePlan *plan, bool encode_maps) {
    if (p.a.M < 1 || p.a.M > WL_DECODE_MAX_M || p.a.K < 8 || p.a.nseg < 1 || num_sms < 1) return WL_ERR_UNSUPPORTED;
    const int NT = (p.a.M + 7) / 8;
    if ((size_t)8 * NT * p.a.t_ld > (size_t)kDecodeTMaxFloats) return WL_ERR_UNSUPPORTED;

    int blocks = 0, max_r = 0;
    bool any_r = false, v_ok = true;
    p.a.u_bulk = 1;
    for (int i = 0; i < p.a.nseg; ++i) {
        DecodeSeg &sg = p.a.seg[i];
        sg.blk_begin = blocks;
        sg.cta_begin = 0;
        blocks += seg_blocks(sg);
        if (sg.r > 0) {
            any_r = true;
            max_r = sg.r > max_r ? sg.r : max_r;
            if (sg.r % 8 != 0 || !aligned_to(sg.U, 16)) p.a.u_bulk = 0;
            if (sg.r % 8 != 0 || !aligned_to(sg.V, 16)) v_ok = false;  // staging and ldmatrix need both
        }
    }
    if (!any_r) {
        p.a.u_bulk = 0;
        v_ok = false;
    }
    p.a.total_blocks = blocks;
    const int grid = blocks < num_sms ? blocks : num_sms;

    // Ring slots: each warp's share of a block's K chunks, at most four chunks.
    const int nchunks = (p.a.K + CK - 1) / CK;
    const int per_warp = (nchunks + NW - 1) / NW;
    p.a.slot_chunks = per_warp < 1 ? 1 : (per_warp > kDecodeMaxSlotChunks ? kDecodeMaxSlotChunks : per_warp);
    p.a.w3d = (p.a.K % CK == 0 && p.a.slot_chunks >= 2) ? 1 : 0;

    wl_status st;
    for (int i = 0; encode_maps && i < p.a.nseg; ++i) {
        const DecodeSeg &sg = p.a.seg[i];
        if ((st = encode_map_2d(&p.tm_w[i], sg.W0, p.a.K, sg.N, p.a.K, CK, BR)) != WL_OK) return st;
        if (p.a.w3d && (st = encode_map_3d(&p.tm_w3[i], sg.W0, CK, sg.N, p.a.K / CK, (uint64_t)p.a.K * 2, CK * 2, CK,
                                         BR, p.a.slot_chunks)) != WL_OK)
            return st;
        if (p.a.u_bulk && sg.r > 0 && (st = encode_map_2d(&p.tm_u[i], sg.U, sg.r, sg.N, sg.r, CK, BR)) != WL_OK)
            return st;
    }

    // T mode.  Local when the V rows any one CTA needs stay small, with the
    // CTAs first shared out among the projections (then a CTA needs one V).
    // Fused local T (rank <= 32, V and U staged, one projection with a delta
    // per CTA) reads V in the W0 MMAs' shadow, so when a CTA has at most two
    // blocks it takes a larger V rather than the grid-wide exchange.
    p.a.seg_split = 0;
    p.a.t_mode = kTNone;
    p.a.t_fused = 0;
    bool fusable = any_r && v_ok && p.a.u_bulk && max_r <= kDecodeFusedMaxRank && p.a.M <= 8;
    size_t worst = 0;
    if (any_r) {
        if (blocks > grid && p.a.nseg > 1) {
            split_ctas(p.a, grid);
            p.a.seg_split = 1;
        }
        p.a.t_mode = kTLocal;
        int most = 0;
        for (int c = 0; c < grid; ++c) {
            int lo, hi;
            cta_blocks(p.a, c, grid, lo, hi);
            size_t bytes = 0;
            int touched = 0;
            for (int i = 0; i < p.a.nseg; ++i)
                if (seg_touched(p.a.seg[i], lo, hi)) {
                    bytes += (size_t)p.a.K * p.a.seg[i].r * 2;
                    ++touched;
                }
            worst = bytes > worst ? bytes : worst;
            most = hi - lo > most ? hi - lo : most;
            if (touched > 1) fusable = false;
        }
        const size_t local_max = (fusable && most <= 2) ? kFusedLocalVBytes : kLocalVBytes;
        if (worst > local_max) {
            p.a.t_mode = kTGrid;
            p.a.seg_split = 0;
            fusable = false;
        }
    }

    bool done = false;
    for (int attempt = 0; !done; ++attempt) {
        if (attempt > 0) {
            // a local-mode V that no layout stages: the grid-wide exchange instead
            if (attempt > 1 || p.a.t_mode != kTLocal || worst <= kLocalVBytes) return WL_ERR_UNSUPPORTED;
            p.a.t_mode = kTGrid;
            p.a.seg_split = 0;
            fusable = false;
        }
        int max_blocks = 0;
        size_t v_bytes = 0, u_bytes = 0;
        for (int c = 0; c < grid; ++c) {
            int lo, hi;
            cta_blocks(p.a, c, grid, lo, hi);
            max_blocks = hi - lo > max_blocks ? hi - lo : max_blocks;
            size_t bytes = 0;
            for (int i = 0; i < p.a.nseg; ++i) {
                int k0, k1;
                v_range(p.a, i, c, grid, lo, hi, k0, k1);
                bytes += (size_t)(k1 - k0) * p.a.seg[i].r * 2;
            }
            v_bytes = bytes > v_bytes ? bytes : v_bytes;
            size_t ub = 0;
            for (int i = 0; i < p.a.nseg; ++i) {
                if (p.a.seg[i].r == 0) continue;
                int b0, b1;
                seg_block_range(p.a.seg[i], lo, hi, b0, b1);
                ub += (size_t)(b1 - b0) * BR * p.a.seg[i].r * 2;
            }
            u_bytes = ub > u_bytes ? ub : u_bytes;
        }
        // the staged rows plus, for a ragged K, room for the rows past the
        // last one that a 16-row k-step reads (and masks)
        const size_t vb = v_bytes + (p.a.K % 16 ? 16 * (size_t)max_r * 2 : 0);
        // grid mode: partial sums in step 1, the reduction in step 2, T loaded in
        // step 3, where the U part of block 0 runs
        p.a.lag = p.a.t_mode == kTGrid ? kDecodeMaxLag : 0;
        p.a.x_ld = p.a.K + 8;

        // Shared memory: the compact variant (two CTAs per SM) for calls whose
        // per-CTA stream is short, when x fits beside a one-slot ring; otherwise
        // the full-size one.  Within the budget: x, then the staged V rows, then
        // more ring slots (up to 192 KB of ring).
        const size_t cta_bytes = (size_t)max_blocks * BR * ((size_t)p.a.K + (size_t)max_r) * 2;
        for (int pass = 0; pass < 2 && !done; ++pass) {
            const bool small = pass == 0;
            if (small && cta_bytes > kSmallCtaBytes) continue;
            const uint32_t budget = small ? kSmallSmem : kDecodeMaxSmem;
            p.a.slots = 1;
            p.a.x_smem = 1;
            p.a.v_stage = 0;
            p.a.v_bytes = 0;
            p.a.v_in_ring = 0;
            p.a.u_stage = 0;
            p.a.u_bytes = 0;
            p.a.t_fused = 0;
            if (smem_layout(p.a, NT).total > budget) {
                if (small) continue;
                p.a.x_smem = 0;
            }
            // Most ring slots that fit the budget with the current choices.
            auto grow_slots = [&]() {
                p.a.slots = 1;
                while (p.a.slots < kDecodeMaxSlots) {
                    ++p.a.slots;
                    const SmemLayout Lg = smem_layout(p.a, NT);
                    if (Lg.total > budget || Lg.ring_bytes > kMaxRingBytes) {
                        --p.a.slots;
                        break;
                    }
                }
            };
            if (fusable && v_bytes > 0 && p.a.x_smem) {
                // fused local T: V and U rows in their own regions
                p.a.t_fused = 1;
                p.a.v_stage = 1;
                p.a.v_bytes = (int)vb;
                p.a.u_stage = 1;
                p.a.u_bytes = (int)u_bytes;
                if (smem_layout(p.a, NT).total <= budget) {
                    grow_slots();
                    plan->small = small ? 1 : 0;
                    done = true;
                    continue;
                }
                p.a.t_fused = 0;
                p.a.v_stage = 0;
                p.a.v_bytes = 0;
                p.a.u_stage = 0;
                p.a.u_bytes = 0;
            }
            if (v_ok && v_bytes > 0) {
                p.a.v_stage = 1;
                p.a.v_bytes = (int)vb;
                p.a.v_in_ring = 0;
                int own_slots = 0;
                if (smem_layout(p.a, NT).total <= budget) {
                    grow_slots();
                    own_slots = p.a.slots;
                }
                // or in the ring's last slot level, when that holds them and
                // leaves more slots for the stream
                p.a.v_in_ring = 1;
                grow_slots();
                const uint32_t level = (uint32_t)NW * p.a.slot_chunks * kDecodeChunkBytes;
                const bool ring_ok = p.a.slots >= 2 && vb <= level && smem_layout(p.a, NT).total <= budget;
                if (!(ring_ok && p.a.slots > own_slots)) {
                    p.a.v_in_ring = 0;
                    if (own_slots > 0) {
                        p.a.slots = own_slots;
                    } else {
                        p.a.v_stage = 0;
                        p.a.v_bytes = 0;
                    }
                }
            }
            // The compact variant only with V staged: without it T is formed
            // element by element on the CUDA cores, far slower than the
            // full-size variant's staged rows.
            if (small && v_ok && v_bytes > 0 && !p.a.v_stage) continue;
            if (!p.a.v_stage) grow_slots();
            if (small && p.a.u_bulk && u_bytes > 0 && !p.a.v_in_ring) {
                // the compact variant's ring is shallow: U rides outside it
                const int slots = p.a.slots;
                p.a.u_stage = 1;
                p.a.u_bytes = (int)u_bytes;
                p.a.slots = 1;
                if (smem_layout(p.a, NT).total > budget) {
                    p.a.u_stage = 0;
                    p.a.u_bytes = 0;
                    p.a.slots = slots;
                } else {
                    grow_slots();
                }
            }
            if (smem_layout(p.a, NT).total > budget) return WL_ERR_UNSUPPORTED;
            plan->small = small ? 1 : 0;
            done = true;
        }
        // local T over a large V only with the rows staged
        if (done && p.a.t_mode == kTLocal && worst > kLocalVBytes && !p.a.v_stage) done = false;
    }
    plan->grid = grid;
    plan->smem = smem_layout(p.a, NT).total;
    plan->tpart_bytes = p.a.t_mode == kTGrid ? (size_t)(grid + 1) * p.a.M * p.a.t_ld * sizeof(float) : 0;
    return WL_OK;
}

template <int NT, bool XS, bool SMALL, int FT>
static cudaError_t launch_decode_v(const DecodeParams &p, const DecodePlan &plan, cudaStream_t stream) {
    // Opt in to the large shared-memory carve-out once per device: both
    // variants run with all of the SM's shared memory configured, so the
    // compact one can hold two CTAs (of consecutive calls) per SM.
    static std::atomic<bool> attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_done[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(decode_kernel<NT, XS, SMALL, FT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kDecodeMaxSmem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(decode_kernel<NT, XS, SMALL, FT>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        attr_done[dev].store(true, std::memory_order_release);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.grid);
    cfg.blockDim = dim3(NTH);
    cfg.dynamicSmemBytes = plan.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_kernel<NT, XS, SMALL, FT>, p);
}

template <int NT>
static cudaError_t launch_decode_nt(const DecodeParams &p, const DecodePlan &plan, cudaStream_t stream) {
    if (plan.small)  // the planner takes the compact variant only with x in shared memory
        return p.a.x_smem ? launch_decode_v<NT, true, true, 0>(p, plan, stream) : cudaErrorInvalidValue;
    return p.a.x_smem ? launch_decode_v<NT, true, false, 0>(p, plan, stream)
                    : launch_decode_v<NT, false, false, 0>(p, plan, stream);
}

// Fused local T: M <= 8, x in shared memory, one or two 16-column tiles of the rank.
template <int FT>
static cudaError_t launch_decode_fused(const DecodeParams &p, const DecodePlan &plan, cudaStream_t stream) {
    return plan.small ? launch_decode_v<1, true, true, FT>(p, plan, stream)
                      : launch_decode_v<1, true, false, FT>(p, plan, stream);
}

cudaError_t launch_decode(const DecodeParams &p, const DecodePlan &plan, cudaStream_t stream) {
    if (p.a.t_fused) {
        if (p.a.M > 8 || !p.a.x_smem) return cudaErrorInvalidValue;
        int max_r = 0;
        for (int i = 0; i < p.a.nseg; ++i) max_r = p.a.seg[i].r > max_r ? p.a.seg[i].r : max_r;
        if (max_r <= 16) return launch_decode_fused<1>(p, plan, stream);
        if (max_r <= 2 * 16) return launch_decode_fused<2>(p, plan, stream);
        return cudaErrorInvalidValue;
    }
    if (p.a.M <= 8) return launch_decode_nt<1>(p, plan, stream);
    if (p.a.M <= 16) return launch_decode_nt<2>(p, plan, stream);
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
