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
// still runs: its whole share of W0 (each lane copies, with 16-byte cp.async,
// exactly the A fragments it will use -- rows g and g + 8 of every block, eight
// consecutive columns of every k-group -- into a region only it reads, so the
// reads are conflict-free and need no barrier), the scales of its outputs, and,
// by bulk copy, the V rows of its slice and the U rows of its group.  The
// eight columns a lane holds are the logical columns 2q, 2q+1, 2q+8, 2q+9 of
// the k-group's first MMA and the same of its second -- a fixed permutation of
// K inside the k-group, applied identically to x (so every dot product is
// unchanged).  A call whose staging fits in half an SM's shared memory leaves
// room for the next call's CTAs, which then stage their weights during this
// call; the CTAs of a launch also pull the following call's weights into L2
// when the caller names them (cross-call prefetch).
//
// Arithmetic.  m16n8k16 MMAs (bf16 in, fp32 accumulate): A = 16 W0 rows from
// the lane's staged fragments, B = x (tokens as the MMA's N) from the slice of x staged in
// shared memory after the wait.  T = V^T x is formed on the same x fragments,
// with A = V^T read by ldmatrix.trans from the staged V rows in the same
// column permutation.  Each warp's partial sums go to shared memory and are
// added in warp order; with c > 1 the CTAs of the cluster then read one
// another's sums over distributed shared memory (fixed CTA order), every CTA
// forms the whole T, and CTA k writes the k-th share of the group's outputs:
// y = bf16_rn(s * z + sum_j U[n][j] T[m][j]), the low-rank product on the
// CUDA cores in fp32.  No atomics: results are reproducible.
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
constexpr uint32_t kRowsSmemMax = 220 * 1024;   // one CTA per SM

__device__ __forceinline__ uint64_t evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// 16 bytes global -> shared without the register file (zeros when src_bytes
// is 0; nothing is then read), with an L2 eviction hint.
__device__ __forceinline__ void cp_async16(void *dst, const void *src, uint32_t src_bytes, uint64_t pol) {
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(smem_addr(dst)),
                 "l"(src), "r"(src_bytes), "l"(pol)
                 : "memory");
}

__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}

// Waits for every cp.async this thread has issued.
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7},"
        " {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&a)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                 : "r"(addr));
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// A float in the shared memory of CTA `rank` of this cluster, at the offset
// `local` has in this CTA.
__device__ __forceinline__ float ld_cluster_f32(const float *local, uint32_t rank) {
    uint32_t ra;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_addr(local)), "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
    return v;
}

// Row of the staged V slice that lane (by its ldmatrix row index lk = 0..15)
// addresses for the first MMA of a k-group (the second adds 4): logical column
// 2q + e of the MMA is physical column 8q + e, and 2q + 8 + e is 8q + 2 + e.
__host__ __device__ __forceinline__ int rows_phys_k(int lk) {
    return lk < 8 ? 8 * (lk >> 1) + (lk & 1) : 8 * ((lk - 8) >> 1) + 2 + (lk & 1);
}

}  // namespace

// Shared memory of a launch (bytes, 128-byte aligned regions).  The W0
// staging region holds, once every warp is past the MMAs, the warps' partial
// sums (z, then T).
__host__ __device__ inline uint32_t rows_rz_bytes(const RowsParams &p) {
    const int NT = p.M > 8 ? 2 : 1;
    return ((uint32_t)p.nb_max * RW * 32u * NT * 16u + 127u) & ~127u;
}

__host__ __device__ inline void rows_layout(RowsParams &p) {
    const int NT = p.M > 8 ? 2 : 1;
    const int rt = (p.r_max + 15) / 16;
    auto al = [](uint32_t v) { return (v + 127u) & ~127u; };
    const uint32_t w_bytes = (uint32_t)p.ks * p.nb_max * 32u;  // 16 rows x 2 bytes per column and block
    const uint32_t red_bytes = rows_rz_bytes(p) + al((uint32_t)RW * rt * 32u * NT * 16u);
    uint32_t o = 0;
    p.off_w = o;
    o += al(w_bytes > red_bytes ? w_bytes : red_bytes);
    p.off_v = o;
    o += al((uint32_t)p.ks * p.r_max * 2u + 32u);  // + room for the 16-column tile's reads past r
    p.off_u = o;
    o += al((uint32_t)p.nb_max * 16u * p.r_max * 2u + 32u);
    p.off_x = o;
    o += al((uint32_t)p.M * (p.ks + kRowsXPad) * 2u);
    p.off_zc = o;
    o += al((uint32_t)p.nb_max * 16u * p.M * 4u);
    p.off_tc = o;
    o += al((uint32_t)p.M * p.r_max * 4u);
    p.off_tf = o;
    o += al((uint32_t)p.M * p.r_max * 4u);
    p.off_s = o;
    o += al((uint32_t)p.nb_max * 16u * 4u);
    p.off_bar = o;
    o += 16u;
    p.smem = o;
}

template <int NT, int NB, int RT>
__global__ void __launch_bounds__(RTH, 2) rows_kernel(const __grid_constant__ RowsParams P) {
    pdl_launch_dependents();
    extern __shared__ __align__(128) uint8_t sm[];
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

    __nv_bfloat16 *vs = reinterpret_cast<__nv_bfloat16 *>(sm + P.off_v);  // [kw][r]
    const __nv_bfloat16 *us = reinterpret_cast<const __nv_bfloat16 *>(sm + P.off_u);  // [rows][r]
    __nv_bfloat16 *xs = reinterpret_cast<__nv_bfloat16 *>(sm + P.off_x);  // [M][ks + pad]
    float *zc = reinterpret_cast<float *>(sm + P.off_zc);    // [16 * nb][M]: this CTA's sums over its slice
    float *tc = reinterpret_cast<float *>(sm + P.off_tc);    // [M][r]: this CTA's T over its slice
    float *tf = reinterpret_cast<float *>(sm + P.off_tf);    // [M][r]: T
    float *ss = reinterpret_cast<float *>(sm + P.off_s);     // scales of this CTA's outputs
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + P.off_bar);
    const int xld = P.ks + kRowsXPad;

    if (tid == 0) {
        mbar_init(bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    // V rows of the slice and U rows of the group
    if (tid == 0 && r > 0) {
        const uint32_t vb = (uint32_t)kw * r * 2u, ub = (uint32_t)rows * r * 2u;
        mbar_arrive_expect_tx(bar, vb + ub);
        bulk_load(vs, S.V + (size_t)k0 * r, vb, bar);
        bulk_load(const_cast<__nv_bfloat16 *>(us), S.U + (size_t)row0 * r, ub, bar);
    }
    // the following call's weights into L2
    if (tid == 32) l2_prefetch_share(P.pf, blockIdx.x, gridDim.x);

    // This warp's k-groups of the slice; the lane's staged fragments: for
    // k-group kl, block b and half h (rows g, g + 8) the 16 bytes at
    // wst + ((kl * nb + b) * 2 + h) * 512 + lane * 16.
    const int nkg = (kw + KG - 1) / KG;
    const int kgA = (warp * nkg) / RW;
    const int nkw = ((warp + 1) * nkg) / RW - kgA;
    uint8_t *wst = sm + P.off_w + (size_t)kgA * nb * 1024u + lane * 16u;
    {
        const uint64_t pol = evict_first_policy();
        const __nv_bfloat16 *wsrc = S.W0 + (size_t)(row0 + g) * K + k0 + (size_t)kgA * KG + 8 * q;
        for (int kl = 0; kl < nkw; ++kl) {
            const bool cv = (kgA + kl) * KG + 8 * q < kw;
            for (int b = 0; b < nb; ++b)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const bool v = cv && b * 16 + 8 * h + g < rows;
                    const void *src = v ? wsrc + (size_t)(b * 16 + 8 * h) * K + kl * KG : (const void *)S.W0;
                    cp_async16(wst + ((kl * nb + b) * 2 + h) * 512u, src, v ? 16u : 0u, pol);
                }
        }
    }
    // The outputs this CTA writes: rows [er0, er1) of the group, every token;
    // their scales.
    const int er0 = (crank * rows) / c, er1 = ((crank + 1) * rows) / c;
    const int nout = (er1 - er0) * M;
    if (tid < er1 - er0) cp_async4(ss + tid, S.s + row0 + er0 + tid);

    pdl_wait_primary();  // the previous kernel is done: x is ready, y is ours
    {
        const int vpr = kw / 8;  // 16-byte vectors per row of the slice
        for (int i = tid; i < M * vpr; i += RTH) {
            const int m = i / vpr, v = i - m * vpr;
            *reinterpret_cast<uint4 *>(xs + (size_t)m * xld + v * 8) =
                __ldg(reinterpret_cast<const uint4 *>(P.x + (size_t)m * K + k0 + v * 8));
        }
    }
    cp_async_wait_all();
    __syncthreads();  // x staged; every thread's copies (its fragments, the scales) landed
    bool ok = true;
    if (r > 0) ok = !__syncthreads_or(!mbar_wait(bar, 0, P.status, P.timeout_ns));

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
    const bool do_t = r > 0 && ok;

    for (int kl = 0; kl < nkw; ++kl) {
        const int col = (kgA + kl) * KG;  // slice-relative
        const bool cv = col + 8 * q < kw;
        uint4 bx[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int n = nt * 8 + g;
            bx[nt] = (cv && n < M) ? *reinterpret_cast<const uint4 *>(xs + (size_t)n * xld + col + 8 * q)
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
                const uint4 lo = *reinterpret_cast<const uint4 *>(wst + ((kl * nb + b) * 2) * 512u);
                const uint4 hi = *reinterpret_cast<const uint4 *>(wst + ((kl * nb + b) * 2 + 1) * 512u);
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

    __syncthreads();  // every warp is past its staged fragments: the region takes the partial sums
    float4 *rz = reinterpret_cast<float4 *>(sm + P.off_w);                     // [nb][RW][32][NT]
    float4 *rtb = reinterpret_cast<float4 *>(sm + P.off_w + rows_rz_bytes(P));  // [RW][rt][32][NT]
    // ---- this warp's partial sums, then the CTA's (warp order) ----
#pragma unroll
    for (int b = 0; b < NB; ++b)
        if (b < nb)  // the region holds the call's largest group, which may be below NB
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                rz[((b * RW + warp) * 32 + lane) * NT + nt] =
                    make_float4(acc[b][nt][0], acc[b][nt][1], acc[b][nt][2], acc[b][nt][3]);
    if (r > 0) {
#pragma unroll
        for (int jt = 0; jt < RT; ++jt)
            if (jt < rt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    rtb[((warp * rt + jt) * 32 + lane) * NT + nt] =
                        make_float4(act[jt][nt][0], act[jt][nt][1], act[jt][nt][2], act[jt][nt][3]);
    }
    __syncthreads();
    // fragment element (row ρ, token column cc) of a 16 x 8 tile: lane
    // (ρ & 7) * 4 + (cc >> 1), element (ρ >> 3) * 2 + (cc & 1)
    for (int e = tid; e < nb * 16 * M; e += RTH) {
        const int row = e / M, m = e - row * M;
        const int b = row >> 4, rr = row & 15, nt = m >> 3, cc = m & 7;
        const int fl = (rr & 7) * 4 + (cc >> 1), fe = (rr >> 3) * 2 + (cc & 1);
        float z = 0.f;
#pragma unroll
        for (int w = 0; w < RW; ++w) z += reinterpret_cast<const float *>(&rz[((b * RW + w) * 32 + fl) * NT + nt])[fe];
        zc[e] = z;
    }
    for (int e = tid; e < M * r; e += RTH) {
        const int m = e / r, j = e - m * r;
        const int jt = j >> 4, jr = j & 15, nt = m >> 3, cc = m & 7;
        const int fl = (jr & 7) * 4 + (cc >> 1), fe = (jr >> 3) * 2 + (cc & 1);
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < RW; ++w) t += reinterpret_cast<const float *>(&rtb[((w * rt + jt) * 32 + fl) * NT + nt])[fe];
        tc[e] = t;
    }
    // ---- the cluster's sums: T in full, z of this CTA's outputs ----
    if (c > 1)
        cluster_sync_all();  // every CTA's sums are in its shared memory
    else
        __syncthreads();
    for (int e = tid; e < M * r; e += RTH) {
        float t = 0.f;
        if (c > 1) {
            for (int k = 0; k < c; ++k) t += ld_cluster_f32(tc + e, (uint32_t)k);
        } else {
            t = tc[e];
        }
        tf[e] = t;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int e = tid + i * RTH;
        if (e < nout) {
            const int row = er0 + e / M, m = e - (e / M) * M;
            float z = 0.f;
            if (c > 1) {
                for (int k = 0; k < c; ++k) z += ld_cluster_f32(zc + row * M + m, (uint32_t)k);
            } else {
                z = zc[row * M + m];
            }
            float dlt = 0.f;
            const __nv_bfloat16 *ur = us + (size_t)row * r;
            const float *tr = tf + (size_t)m * r;
            for (int j = 0; j < r; j += 8) {
                const uint4 uv = *reinterpret_cast<const uint4 *>(ur + j);
                const float4 ta = *reinterpret_cast<const float4 *>(tr + j);
                const float4 tb = *reinterpret_cast<const float4 *>(tr + j + 4);
                dlt = fmaf(bf16lo(uv.x), ta.x, dlt);
                dlt = fmaf(bf16hi(uv.x), ta.y, dlt);
                dlt = fmaf(bf16lo(uv.y), ta.z, dlt);
                dlt = fmaf(bf16hi(uv.y), ta.w, dlt);
                dlt = fmaf(bf16lo(uv.z), tb.x, dlt);
                dlt = fmaf(bf16hi(uv.z), tb.y, dlt);
                dlt = fmaf(bf16lo(uv.w), tb.z, dlt);
                dlt = fmaf(bf16hi(uv.w), tb.w, dlt);
            }
            if (ok) S.y[(size_t)m * N + row0 + row] = __float2bfloat16_rn(fmaf(ss[row - er0], z, dlt));
        }
    }
    if (c > 1) cluster_sync_all();  // no CTA leaves while another may still read its shared memory
    // after a timed-out wait, the copies still in flight land before the CTA exits
    if (!ok && tid == 0) mbar_wait(bar, 0, P.status, 1000000ull);
}

// ------------------------------------------------------------------ host ---
namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

wl_status plan_rows(RowsParams &p, int M, int K, const wl_proj *projs, int P, int num_sms) {
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
    // (the next call's CTAs take the other half) come first; among those, or
    // else among the rest, the one with the fewest bytes per CTA (its W0
    // blocks over its slice plus its V slice) wins, ties keeping the smaller
    // cluster.
    bool found = false, best_half = false;
    size_t best = 0;
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
        size_t cost = 0;
        RowsParams t = p;
        for (int i = 0; i < nseg; ++i) {
            const int nb = (blocks[i] + ngrp[i] - 1) / ngrp[i];
            t.seg[i].nb = nb;
            t.seg[i].grp_begin = groups;
            groups += (blocks[i] + nb - 1) / nb;
            nbmax = nb > nbmax ? nb : nbmax;
            const size_t bytes = (size_t)nb * 16 * ks * 2 + (size_t)ks * t.seg[i].r * 2;
            cost = bytes > cost ? bytes : cost;
        }
        if (nbmax > kRowsMaxBlocks) continue;
        t.c = c;
        t.ks = ks;
        t.ngroups = groups;
        t.nb_max = nbmax;
        rows_layout(t);
        if (t.smem > kRowsSmemMax) continue;
        const bool half = t.smem <= kRowsSmemHalf;
        if (!found || (half && !best_half) || (half == best_half && cost < best)) {
            found = true;
            best_half = half;
            best = cost;
            cand = t;
        }
    }
    if (!found) return WL_ERR_UNSUPPORTED;
    p = cand;
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
