// Row-stream decode kernel: the theta-bundle linear y = s (.) (W0 x) + U (V^T x)
// for short calls (up to 16 tokens, a few MB of weights), where the time of a
// call is set by latency -- the wait for the previous kernel, one round trip
// for x, the reductions -- rather than by the HBM stream.
//
// Work split.  The output rows of each projection are cut into 16-row blocks
// and the blocks into row groups of at most kRowsMaxBlocks; a row group is
// owned by a cluster of c CTAs (c = 1, 2 or 4), CTA k of the cluster taking
// the k-th slice of K.  The eight warps of a CTA split the slice's 32-column
// k-groups evenly and each covers all blocks of the group.
//
// Staging.  Everything a CTA reads that is a weight is requested before the
// wait for the previous kernel (griddepcontrol.wait), i.e. while that kernel
// still runs: its whole share of W0 and, by bulk copy, the V rows of its slice
// and the U rows of its group.  Each warp copies its k-groups of W0 with one
// TMA tile per k-group (32 columns x the group's rows, no swizzle): the tile
// lands as 64-byte rows, so the 16 bytes lane (g, q) needs -- eight
// consecutive columns of row g (or g + 8) of a block -- sit at 16 * lane in
// each 512-byte half-block, and every lane reads its own fragments
// conflict-free.  Those eight columns are the logical columns 2q, 2q+1, 2q+8,
// 2q+9 of the k-group's first MMA and the same of its second -- a fixed
// permutation of K inside the k-group, applied identically to x (so every dot
// product is unchanged).  A call whose staging fits in half an SM's shared
// memory leaves room for the next call's CTAs, which then stage their weights
// during this call; the CTAs of a launch also pull the following call's
// weights into L2 when the caller names them (cross-call prefetch).
//
// Arithmetic.  m16n8k16 MMAs (bf16 in, fp32 accumulate): A = 16 W0 rows from
// the lane's staged fragments, B = x (tokens as the MMA's N), which each warp
// stages for its own k-groups after the wait (no CTA barrier).  T = V^T x is
// formed on the same x fragments, with A = V^T read by ldmatrix.trans from
// the staged V rows in the same column permutation.  Since U T is the sum of
// U T_w over the warps' partial T_w, each warp multiplies its own T_w (split
// into bf16 high and low parts, fp32-level accuracy) by the U rows of every
// block on the tensor cores, so T is never gathered.  The warps' sums of
// W0 x and of U T are added in warp order after one CTA barrier; with c > 1
// each CTA pushes its slice's sums into the shared memory of the CTA that
// writes each output, and after one cluster barrier those are added in rank
// order: y = bf16_rn(s * z + U T).  No atomics: results are reproducible.
//
// Prior art: the custom-op kernel on "Quality (Gemma 4 31B)", "Kernel
// optimizations", custom-op path (128-bit loads, warp-level reductions,
// cooperative V^T x, memory-bound at small dimensions).  Here the per-row dot
// products run on the tensor cores from register-held fragments, K is split
// over CTA clusters, and consecutive calls overlap through programmatic
// dependent launch and the L2 prefetch of the following call's weights.
#include <atomic>
#include <cstring>

#include "wl_common.cuh"
#include "wl_internal.h"
#include "wl_prefetch.cuh"

namespace wl {

namespace {

constexpr int RW = kRowsWarps;
constexpr int RTH = kRowsThreads;
constexpr int KG = kRowsKGroup;
constexpr uint32_t kRowsSmemHalf = 110 * 1024;  // two CTAs per SM: this call's and the next one's
constexpr uint32_t kRowsSmemMax = 226 * 1024;   // one CTA per SM

__device__ __forceinline__ uint64_t evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ void tma_tile_2d(void *dst, const void *tmap, int c0, int c1, uint64_t *bar,
                                            uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(smem_addr(bar)), "l"(pol)
        : "memory");
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7},"
        " {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&a)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&a)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                 : "r"(addr));
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Stores (a, b) into the shared memory of CTA `rank` of this cluster, at the
// offset `local` has in this CTA (8-byte aligned).
__device__ __forceinline__ void st_cluster_f32x2(float *local, uint32_t rank, float a, float b) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_addr(local)), "r"(rank));
    asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(ra), "f"(a), "f"(b) : "memory");
}

// Row of the staged V slice that lane (by its ldmatrix row index lk = 0..15)
// addresses for the first MMA of a k-group (the second adds 4): logical column
// 2q + e of the MMA is physical column 8q + e, and 2q + 8 + e is 8q + 2 + e.
__host__ __device__ __forceinline__ int rows_phys_k(int lk) {
    return lk < 8 ? 8 * (lk >> 1) + (lk & 1) : 8 * ((lk - 8) >> 1) + 2 + (lk & 1);
}

}  // namespace

// Shared memory of a launch (bytes, 128-byte aligned regions, from the first
// 1024-byte boundary of the dynamic shared memory).
__host__ __device__ inline int rows_nkw_max(const RowsParams &p) {
    const int nkg = p.ks / KG;
    return (nkg + RW - 1) / RW;  // k-groups of the busiest warp
}

__host__ __device__ inline void rows_layout(RowsParams &p) {
    const int NT = p.M > 8 ? 2 : 1;
    auto al = [](uint32_t v) { return (v + 127u) & ~127u; };
    const uint32_t part = al((uint32_t)p.nb_max * RW * 32u * NT * 16u);  // one fragment set per block and warp
    uint32_t o = 0;
    p.off_w = o;  // W0 tiles: [k-group][block][16 rows][32 columns]
    o += al((uint32_t)p.ks * p.nb_max * 32u);
    p.off_v = o;  // V rows of the slice (+ room for a 16-column tile's reads past r)
    o += al((uint32_t)p.ks * p.r_max * 2u + 32u);
    p.off_u = o;  // U rows of the group, whole 16-row blocks
    o += al((uint32_t)p.nb_max * 16u * p.r_max * 2u + 32u);
    p.off_x = o;  // per warp: [its k-group][token][32 columns] of x
    o += al((uint32_t)RW * rows_nkw_max(p) * p.M * 64u);
    p.off_zc = o;  // per warp and block: W0 x partial sums (fragments); then, with
    o += part;     // clusters, the CTA's sums [16 nb][M]
    p.off_tc = o;  // the same for U T
    o += part;
    p.off_tf = o;  // clusters: [rank][its share of the outputs][M] pairs (z, U T) of every CTA's sums
    o += al((uint32_t)p.c * ((p.nb_max * 16u + p.c - 1) / p.c) * p.M * 8u);
    p.off_s = o;   // scales of the CTA's outputs
    o += al((uint32_t)p.nb_max * 16u * 4u);
    p.off_bar = o;
    o += (1u + RW) * 8u;  // V / U staged; each warp's W0 tiles
    p.smem = o + 1024u;   // + the slack for the 1024-byte alignment
}

template <int NT, int NB, int RT>
__global__ void __launch_bounds__(RTH, 2) rows_kernel(const __grid_constant__ RowsParams P) {
    pdl_launch_dependents();
    // the regions are laid out from the first 1024-byte boundary of the
    // dynamic shared memory (the launch adds the slack)
    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
    const int c = P.c;
    const int crank = (int)(blockIdx.x % (unsigned)c);  // the CTA's rank in its (1-D) cluster
    const int cid = (int)(blockIdx.x / (unsigned)c);
    int sp = 0;
    while (sp + 1 < P.nseg && cid >= P.seg[sp + 1].grp_begin) ++sp;
    const RowsSeg &S = P.seg[sp];
    const int N = S.N, r = S.r, K = P.K, M = P.M;
    const int b0 = (cid - S.grp_begin) * S.nb;
    const int nb = min(S.nb, (N + 15) / 16 - b0);  // >= 1 (the planner makes no empty group)
    const int row0 = b0 * 16;
    const int rows = min(N - row0, nb * 16);
    const int k0 = crank * P.ks;                   // < K (the planner makes no empty slice)
    const int kw = min(K, k0 + P.ks) - k0;         // a multiple of 8
    const int rt = (r + 15) >> 4;

    const __nv_bfloat16 *vs = reinterpret_cast<const __nv_bfloat16 *>(sm + P.off_v);  // [kw][r]
    const __nv_bfloat16 *us = reinterpret_cast<const __nv_bfloat16 *>(sm + P.off_u);  // [16 nb][r]
    float4 *rz = reinterpret_cast<float4 *>(sm + P.off_zc);  // [nb][RW][32][NT]: W0 x
    float4 *rd = reinterpret_cast<float4 *>(sm + P.off_tc);  // [nb][RW][32][NT]: U T
    float *cs = reinterpret_cast<float *>(sm + P.off_tf);    // clusters: [rank][share][M][2]
    float *ss = reinterpret_cast<float *>(sm + P.off_s);     // scales of this CTA's outputs
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + P.off_bar);
    uint64_t *wbar = bar + 1;  // [RW]: each warp's W0 tiles landed

    if (tid == 0) {
        mbar_init(bar, 1);
        for (int w = 0; w < RW; ++w) mbar_init(&wbar[w], 1);
        fence_barrier_init();
    }
    // The U MMAs of the last row read up to 8 elements past its r columns
    // (a 16-column tile of an r % 16 == 8 rank); they meet zero T, but must
    // be finite: clear the 32 bytes after the rows the bulk copy fills.
    if (tid == 64 && r > 0) {
        uint4 *tail = reinterpret_cast<uint4 *>(sm + P.off_u + (size_t)rows * r * 2u);
        tail[0] = tail[1] = make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();
    // V rows of the slice and U rows of the group
    if (tid == 0 && r > 0) {
        const uint32_t vb = (uint32_t)kw * r * 2u, ub = (uint32_t)rows * r * 2u;
        mbar_arrive_expect_tx(bar, vb + ub);
        bulk_load(const_cast<__nv_bfloat16 *>(vs), S.V + (size_t)k0 * r, vb, bar);
        bulk_load(const_cast<__nv_bfloat16 *>(us), S.U + (size_t)row0 * r, ub, bar);
    }
    // This warp's k-groups of the slice, and its W0 tiles: k-group kl (of the
    // warp) is one tile of S.nb blocks (rows past N arrive as zeros), and the
    // 16 bytes lane `lane` uses for block b, half h sit at
    // wst + ((kl * S.nb + b) * 2 + h) * 512 (wst includes the lane's 16 * lane).
    const int nkg = (kw + KG - 1) / KG;
    const int kgA = (warp * nkg) / RW;
    const int nkw = ((warp + 1) * nkg) / RW - kgA;
    const int bb = S.nb;  // blocks per tile
    uint8_t *wbase = sm + P.off_w + (size_t)kgA * bb * 1024u;
    const uint8_t *wst = wbase + lane * 16u;
    if (lane == 0 && nkw > 0) {
        const uint64_t pol = evict_first_policy();
        mbar_arrive_expect_tx(&wbar[warp], (uint32_t)nkw * bb * 1024u);
        for (int kl = 0; kl < nkw; ++kl)
            tma_tile_2d(wbase + (size_t)kl * bb * 1024u, &P.tm_w[sp], k0 + (kgA + kl) * KG, row0, &wbar[warp], pol);
    }
    // The outputs this CTA writes: rows [er0, er1) of the group, every token;
    // their scales into shared memory (the barrier below keeps these loads
    // ahead of the wait for the previous kernel).
    const int er0 = (crank * rows) / c, er1 = ((crank + 1) * rows) / c;
    const int nout = (er1 - er0) * M;
    if (tid < er1 - er0) ss[tid] = __ldg(S.s + row0 + er0 + tid);
    __syncthreads();
    // The copies usually land while the previous kernel still runs: wait for
    // them here, off the path that follows the wait for that kernel.
    bool ok = true;
    if (r > 0) ok = mbar_wait(bar, 0, P.status, P.timeout_ns);
    if (nkw > 0 && !mbar_wait(&wbar[warp], 0, P.status, P.timeout_ns)) ok = false;
    // The following call's weights into L2, once this warp's own copies have
    // landed (the prefetches take the same copy engine).
    if (warp == RW - 1 && lane == 0) l2_prefetch_share(P.pf, blockIdx.x, gridDim.x);

    pdl_wait_primary();  // the previous kernel is done: x is ready, y is ours
    // x: each warp stages the columns of its own k-groups (no CTA barrier),
    // [k-group][token][32 columns]
    __nv_bfloat16 *xw = reinterpret_cast<__nv_bfloat16 *>(sm + P.off_x) + (size_t)warp * rows_nkw_max(P) * M * KG;
    for (int i = lane; i < nkw * M * 4; i += 32) {
        const int kl = i / (M * 4), rem = i - kl * M * 4, m = rem >> 2, qq = rem & 3;
        const int col = (kgA + kl) * KG + 8 * qq;  // slice-relative
        const uint4 v = col < kw ? __ldg(reinterpret_cast<const uint4 *>(P.x + (size_t)m * K + k0 + col))
                                 : make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4 *>(xw + ((size_t)kl * M + m) * KG + 8 * qq) = v;
    }
    __syncwarp();

    float acc[NB][NT][4];
    float act[RT][NT][4];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[b][nt][e] = 0.f;
#pragma unroll
    for (int jt = 0; jt < RT; ++jt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) act[jt][nt][e] = 0.f;
    // ldmatrix.trans addressing of V^T fragments: this lane supplies logical
    // row lk (physical rows_phys_k(lk), + 4 for the second MMA) and the
    // 8-column half lj of the 16-column tile
    const int lk = (lane & 7) + ((lane >> 4) << 3);
    const int lphys = rows_phys_k(lk);
    const int lj = ((lane >> 3) & 1) << 3;
    const uint32_t vs_addr = smem_addr(vs);
    const bool do_t = r > 0;

    for (int kl = 0; kl < nkw; ++kl) {
        const int col = (kgA + kl) * KG;  // slice-relative
        const bool cv = col + 8 * q < kw;
        uint4 bx[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int n = nt * 8 + g;
            bx[nt] = n < M ? *reinterpret_cast<const uint4 *>(xw + ((size_t)kl * M + n) * KG + 8 * q)
                           : make_uint4(0u, 0u, 0u, 0u);
        }
        if (do_t) {
#pragma unroll
            for (int jt = 0; jt < RT; ++jt) {
                if (jt < rt) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        int vrow = col + lphys + 4 * h;
                        if (vrow >= kw) vrow = 0;  // past the slice: any staged row (masked below)
                        uint32_t a[4];
                        ldsm_x4_trans(vs_addr + (uint32_t)(vrow * r + jt * 16 + lj) * 2u, a);
                        if (!cv) a[0] = a[1] = a[2] = a[3] = 0u;  // this lane's chunk is past K
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
                            mma16816(act[jt][nt], a, h ? bx[nt].z : bx[nt].x, h ? bx[nt].w : bx[nt].y);
                    }
                }
            }
        }
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            if (b < nb) {
                const uint4 lo = *reinterpret_cast<const uint4 *>(wst + ((kl * bb + b) * 2) * 512u);
                const uint4 hi = *reinterpret_cast<const uint4 *>(wst + ((kl * bb + b) * 2 + 1) * 512u);
                const uint32_t a1[4] = {lo.x, hi.x, lo.y, hi.y};
                const uint32_t a2[4] = {lo.z, hi.z, lo.w, hi.w};
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    mma16816(acc[b][nt], a1, bx[nt].x, bx[nt].y);
                    mma16816(acc[b][nt], a2, bx[nt].z, bx[nt].w);
                }
            }
        }
    }

    // ---- the low-rank part of this warp: U (T over the warp's k-groups) ----
    // U T = sum over the warps of U T_w, so each warp multiplies its own
    // partial T (fp32, split into bf16 high and low parts) by the U rows of
    // every block; no warp needs the whole T.  T_w's accumulator fragment
    // (rank j as rows, tokens as columns) is moved into the B-operand layout
    // (rank j as the MMA's K) with shuffles: lane (g, q) needs T[2q, 2q+1,
    // 2q+8, 2q+9][token g], held by lanes 8q + (g >> 1) and 8q + 4 + (g >> 1)
    // as elements (g & 1) and 2 + (g & 1).
    float acd[NB][NT][4];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acd[b][nt][e] = 0.f;
    if (do_t) {
        const int src0 = 8 * q + (g >> 1), src1 = src0 + 4;
        const bool odd = g & 1;
#pragma unroll
        for (int jt = 0; jt < RT; ++jt) {
            if (jt < rt) {
                uint32_t bh[NT][2], bl[NT][2];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float v[4];  // T[2q], T[2q+1], T[2q+8], T[2q+9] of token nt * 8 + g
                    const float a0 = __shfl_sync(0xffffffffu, act[jt][nt][0], src0);
                    const float a1 = __shfl_sync(0xffffffffu, act[jt][nt][1], src0);
                    const float a2 = __shfl_sync(0xffffffffu, act[jt][nt][2], src0);
                    const float a3 = __shfl_sync(0xffffffffu, act[jt][nt][3], src0);
                    const float c0 = __shfl_sync(0xffffffffu, act[jt][nt][0], src1);
                    const float c1 = __shfl_sync(0xffffffffu, act[jt][nt][1], src1);
                    const float c2 = __shfl_sync(0xffffffffu, act[jt][nt][2], src1);
                    const float c3 = __shfl_sync(0xffffffffu, act[jt][nt][3], src1);
                    v[0] = odd ? a1 : a0;
                    v[1] = odd ? c1 : c0;
                    v[2] = odd ? a3 : a2;
                    v[3] = odd ? c3 : c2;
                    // rank columns past r are not part of the product
                    const int j0 = jt * 16 + 2 * q;
                    if (j0 >= r) v[0] = 0.f;
                    if (j0 + 1 >= r) v[1] = 0.f;
                    if (j0 + 8 >= r) v[2] = 0.f;
                    if (j0 + 9 >= r) v[3] = 0.f;
                    bh[nt][0] = pack_bf16x2(v[0], v[1]);
                    bh[nt][1] = pack_bf16x2(v[2], v[3]);
                    bl[nt][0] = pack_bf16x2(v[0] - bf16lo(bh[nt][0]), v[1] - bf16hi(bh[nt][0]));
                    bl[nt][1] = pack_bf16x2(v[2] - bf16lo(bh[nt][1]), v[3] - bf16hi(bh[nt][1]));
                }
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    if (b < nb) {
                        // A = U rows 16 b .. 16 b + 15, rank columns 16 jt ..: row lane & 15,
                        // column half lane >> 4 (rows past the group hold anything: their
                        // outputs are never written; columns past r meet zero T)
                        uint32_t a[4];
                        ldsm_x4(smem_addr(us) + (uint32_t)((b * 16 + (lane & 15)) * r + jt * 16 + (lane >> 4) * 8) * 2u, a);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            mma16816(acd[b][nt], a, bh[nt][0], bh[nt][1]);
                            mma16816(acd[b][nt], a, bl[nt][0], bl[nt][1]);
                        }
                    }
                }
            }
        }
    }
#pragma unroll
    for (int b = 0; b < NB; ++b)
        if (b < nb)  // the regions hold the call's largest group, which may be below NB
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                rz[((b * RW + warp) * 32 + lane) * NT + nt] =
                    make_float4(acc[b][nt][0], acc[b][nt][1], acc[b][nt][2], acc[b][nt][3]);
                rd[((b * RW + warp) * 32 + lane) * NT + nt] =
                    make_float4(acd[b][nt][0], acd[b][nt][1], acd[b][nt][2], acd[b][nt][3]);
            }
    ok = !__syncthreads_or(!ok);  // every warp's sums are in

    // Output (row, token) of the group: the eight warps' sums in warp order.
    // Fragment element (row rr, token column cc) of a 16 x 8 tile: lane
    // (rr & 7) * 4 + (cc >> 1), element (rr >> 3) * 2 + (cc & 1).
    auto warp_sums = [&](int row, int m, float &z, float &d) {
        const int b = row >> 4, rr = row & 15, nt = m >> 3, cc = m & 7;
        const int fl = (rr & 7) * 4 + (cc >> 1), fe = (rr >> 3) * 2 + (cc & 1);
        z = d = 0.f;
#pragma unroll
        for (int w = 0; w < RW; ++w) {
            z += reinterpret_cast<const float *>(&rz[((b * RW + w) * 32 + fl) * NT + nt])[fe];
            d += reinterpret_cast<const float *>(&rd[((b * RW + w) * 32 + fl) * NT + nt])[fe];
        }
    };
    if (c == 1) {
        for (int e = tid; e < nout; e += RTH) {
            const int row = e / M, m = e - row * M;
            float z, d;
            warp_sums(row, m, z, d);
            if (ok) S.y[(size_t)m * N + row0 + row] = __float2bfloat16_rn(fmaf(ss[row], z, d));
        }
    } else {
        // Each CTA adds up its warps' sums over its slice for every output of
        // the group and stores them into the shared memory of the CTA that
        // writes that output (slot [its rank]); one cluster-wide barrier
        // later every CTA holds all c slices of its outputs in its own
        // shared memory and adds them in rank order.  Nobody touches another
        // CTA's shared memory after that barrier, so no second one is needed.
        const int share = (rows + c - 1) / c;  // outputs of one rank, at most (rows per rank) * M
        for (int e = tid; e < rows * M; e += RTH) {
            const int row = e / M, m = e - row * M;
            float z, d;
            warp_sums(row, m, z, d);
            int owner = 0;  // the rank whose [er0, er1) holds row
            while (owner + 1 < c && row >= ((owner + 1) * rows) / c) ++owner;
            const int ol = (row - (owner * rows) / c) * M + m;  // its index in the owner's share
            float *slot = cs + ((size_t)crank * share * M + ol) * 2;
            st_cluster_f32x2(slot, (uint32_t)owner, z, d);
        }
        cluster_sync_all();  // every CTA's slices of my outputs are in my shared memory
        for (int e = tid; e < nout; e += RTH) {
            const int row = er0 + e / M, m = e - (e / M) * M;
            float z = 0.f, d = 0.f;
            for (int k = 0; k < c; ++k) {
                const float2 v = *reinterpret_cast<const float2 *>(cs + ((size_t)k * share * M + e) * 2);
                z += v.x;
                d += v.y;
            }
            if (ok) S.y[(size_t)m * N + row0 + row] = __float2bfloat16_rn(fmaf(ss[row - er0], z, d));
        }
    }
    // after a timed-out wait, the copies still in flight land before the CTA exits
    if (!ok && tid == 0 && r > 0) mbar_wait(bar, 0, P.status, 1000000ull);
    if (!ok && lane == 0 && nkw > 0) mbar_wait(&wbar[warp], 0, P.status, 1000000ull);
}

// ------------------------------------------------------------------ host ---
namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

wl_status plan_rows(RowsParams &p, int M, int K, const wl_proj *projs, int P, int num_sms, bool encode_maps) {
    std::memset(&p, 0, sizeof p);
    if (M < 1 || M > 16 || K < 8 || K % 8 != 0 || num_sms < 1) return WL_ERR_UNSUPPORTED;
    int nseg = 0, blocks[kMaxSeg], rmax = 0;
    for (int i = 0; i < P; ++i) {
        const wl_proj &q = projs[i];
        if (q.N == 0) continue;
        if (q.r > kRowsMaxRank || q.r % 8 != 0) return WL_ERR_UNSUPPORTED;
        if (q.r > 0 && (!aligned16(q.U) || !aligned16(q.V))) return WL_ERR_UNSUPPORTED;
        RowsSeg &sg = p.seg[nseg];
        sg.W0 = reinterpret_cast<const __nv_bfloat16 *>(q.W0);
        sg.s = q.s;
        sg.U = reinterpret_cast<const __nv_bfloat16 *>(q.U);
        sg.V = reinterpret_cast<const __nv_bfloat16 *>(q.V);
        sg.y = reinterpret_cast<__nv_bfloat16 *>(q.y);
        sg.N = q.N;
        sg.r = q.r;
        blocks[nseg] = (q.N + 15) / 16;
        rmax = q.r > rmax ? q.r : rmax;
        ++nseg;
    }
    if (nseg == 0) return WL_ERR_UNSUPPORTED;
    p.nseg = nseg;
    p.M = M;
    p.K = K;
    p.r_max = rmax;

    // Over the cluster sizes: the row groups each get at most kRowsMaxBlocks
    // blocks and one CTA of a cluster per slice, with at most one CTA of the
    // call per SM.  Splits whose staging fits in half an SM's shared memory
    // (the next call's CTAs take the other half) come first; then the
    // smallest cluster: a cluster's sums cost two cluster-wide barriers after
    // the wait for the previous kernel, while the staging that more CTAs
    // would share happens before it.
    bool found = false, best_half = false;
    RowsParams cand = p;
    for (int c = 1; c <= kRowsMaxCluster; c *= 2) {
        const int ks = ((K + c - 1) / c + KG - 1) / KG * KG;
        if ((c - 1) * ks >= K) continue;  // a slice would be empty
        const int G = num_sms / c;
        if (G < nseg) continue;
        int ngrp[kMaxSeg], used = 0;
        for (int i = 0; i < nseg; ++i) {
            ngrp[i] = 1;
            ++used;
        }
        while (used < G) {
            int bi = -1, bl = 0;
            for (int i = 0; i < nseg; ++i) {
                if (ngrp[i] >= blocks[i]) continue;
                const int load = (blocks[i] + ngrp[i] - 1) / ngrp[i];
                if (load > bl) {
                    bl = load;
                    bi = i;
                }
            }
            if (bi < 0) break;
            ++ngrp[bi];
            ++used;
        }
        int nbmax = 0, groups = 0;
        RowsParams t = p;
        for (int i = 0; i < nseg; ++i) {
            const int nb = (blocks[i] + ngrp[i] - 1) / ngrp[i];
            t.seg[i].nb = nb;
            t.seg[i].grp_begin = groups;
            groups += (blocks[i] + nb - 1) / nb;
            nbmax = nb > nbmax ? nb : nbmax;
        }
        if (nbmax > kRowsMaxBlocks) continue;
        t.c = c;
        t.ks = ks;
        t.ngroups = groups;
        t.nb_max = nbmax;
        rows_layout(t);
        if (t.smem > kRowsSmemMax) continue;
        const bool half = t.smem <= kRowsSmemHalf;
        // c grows through the loop: a later split replaces the kept one only
        // by fitting in half an SM where the kept one does not
        if (!found || (half && !best_half)) {
            found = true;
            best_half = half;
            cand = t;
        }
    }
    if (!found) return WL_ERR_UNSUPPORTED;
    p = cand;
    for (int i = 0; encode_maps && i < p.nseg; ++i) {
        const wl_status st = encode_map_2d(&p.tm_w[i], p.seg[i].W0, (uint64_t)K, (uint64_t)p.seg[i].N, (uint64_t)K,
                                           KG, (uint32_t)p.seg[i].nb * 16u, false);
        if (st != WL_OK) return st;
    }
    return WL_OK;
}

namespace {

template <int NT, int NB, int RT>
cudaError_t launch_rows_v(const RowsParams &p, cudaStream_t stream) {
    static std::atomic<bool> attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_done[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(rows_kernel<NT, NB, RT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kRowsSmemMax);
        if (e != cudaSuccess) return e;
        attr_done[dev].store(true, std::memory_order_release);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.ngroups * p.c));
    cfg.blockDim = dim3(RTH);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    int na = 1;
    if (p.c > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = (unsigned)p.c;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        na = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, rows_kernel<NT, NB, RT>, p);
}

template <int NT, int NB>
cudaError_t launch_rows_nb(const RowsParams &p, cudaStream_t stream) {
    // 16-column tiles of T the largest rank needs (a rank-0 call takes one)
    if (p.r_max <= 16) return launch_rows_v<NT, NB, 1>(p, stream);
    if (p.r_max <= 32) return launch_rows_v<NT, NB, 2>(p, stream);
    if (p.r_max <= kRowsMaxRank) return launch_rows_v<NT, NB, 4>(p, stream);
    return cudaErrorInvalidValue;
}

template <int NT>
cudaError_t launch_rows_nt(const RowsParams &p, cudaStream_t stream) {
    if (p.nb_max <= 1) return launch_rows_nb<NT, 1>(p, stream);
    if (p.nb_max <= 2) return launch_rows_nb<NT, 2>(p, stream);
    if (p.nb_max <= 4) return launch_rows_nb<NT, 4>(p, stream);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_rows(const RowsParams &p, cudaStream_t stream) {
    if (p.ngroups < 1 || p.c < 1 || p.c > kRowsMaxCluster || p.smem > kRowsSmemMax) return cudaErrorInvalidValue;
    return p.M <= 8 ? launch_rows_nt<1>(p, stream) : launch_rows_nt<2>(p, stream);
}

}  // namespace wl
