// The two-launch decode kernels: a prep launch (V^T x and a permuted copy of
// x) followed by a weight stream.  They serve the NVFP4 shared block (below)
// and, through the persistent ring with bf16 weight tiles, the large bf16
// calls of at most 8 tokens (WL_PATH_RING; the ring section at the end of this
// comment).  The parameter block is shared (Fp4Params; bf16 = 1 for the bf16
// ring, whose "codes" are the bf16 rows, with no scales and tensor scale 1).
//
// Decode with an NVFP4 shared block: y = s (.) (W0 x) + U (V^T x) where W0 is
// stored as FP4 E2M1 codes (two per byte, element 2i in the low nibble of
// byte i), one FP8 E4M3 scale per 16 consecutive elements of a row, and one
// fp32 tensor scale -- 0.5625 bytes per element instead of 2 ("Compression",
// "NVFP4: 3.18x smaller weights": packed 4-bit weights with an e4m3 scale per
// 16 elements, dequantised on the fly).  U, V and s stay as in the bf16 path.
//
// Two launches per call.
//
// prep: T = V^T x (fp32) for every projection with a delta.  CTA (projection,
//   slice) takes kr rows of V: its threads split the rank into 8-column
//   groups (one 16-byte load per row) and the slice's rows, the row partial
//   sums are added in a fixed order; then the last CTA of each group of
//   kFp4GroupSlices slices adds the group's partials in slice order, and the
//   last group adds the group sums in group order (no float atomics, two short
//   serial steps instead of one long one).  The same launch writes x as f16 in
//   the permuted order the weight stream reads (below).
//
// The weight stream's arithmetic (both variants).  Within a 128-column
// k-group, lane (g, q) of a warp owns columns 32q .. 32q + 31 of rows g and
// g + 8 of a 16-row block: 16 bytes of codes and two scale bytes per row.  It
// expands them with the hardware E2M1 -> f16 and E4M3 -> f16 conversions and
// one f16 multiply per pair (an E2M1 value times an E4M3 scale is exact in
// f16) and runs eight m16n8k16 MMAs (f16 in, fp32 accumulate): MMA i takes the
// lane's elements 4i .. 4i + 3 as its logical columns 2q, 2q + 1, 2q + 8,
// 2q + 9 -- a fixed permutation of K inside the k-group, which the prep launch
// applies to x once, laid out so that each lane reads its 32 values of x as
// four conflict-free 16-byte pieces:
//     xq[kg][t][m][q][j] = x[m][128 kg + 32 q + 8 t + j]     (t, q < 4; j < 8)
// with Mp token rows (M, rounded up to even above 1; the extra row is zero).
// U T runs on the tensor cores too: A = 16 U rows, B = T split into bf16 high
// and low parts (two MMAs), so the low-rank product keeps fp32-level accuracy.
// Per block the eight warps' fragments are added in warp order and
//     y = bf16_rn((s * tensor_scale) * z + U T).
// The tensor scale multiplies s (both are per-row factors of the W0 product).
//
// ring (K % 256 == 0 and every rank <= 256): a persistent launch, one CTA per
//   SM, 8 consumer warps and one producer warp.  A projection's work is a
//   sequence of units: for each 16-row block, its stages (2048 columns: the
//   codes as one TMA box of 16 rows x 1024 bytes, the scales as 16 rows x 128
//   bytes, and the stage's slice of the permuted x by a bulk copy) and then,
//   when r > 0, one U unit (16 rows x 2r bytes).  Every box is 16 long rows:
//   a tensor copy's cost grows with its row count, and boxes of short rows
//   (64 bytes and less) held the stream far below the HBM rate.  The units of the
//   whole call are cut into one contiguous, equal range per CTA, so every CTA
//   streams the same number of bytes; a block whose units fall into two or
//   more CTAs' ranges is finished by the last of them to arrive (a counter per
//   block), which adds the CTAs' partial sums in CTA order.  The producer
//   requests the whole ring of weight tiles before the wait for the prep
//   launch, then the x slices of those units, then keeps the ring full.  Warp
//   w takes k-groups w and w + 8 of every stage and rank columns 32w .. 32w + 31 of every
//   U unit (lane q eight consecutive ones, the same permutation of the rank
//   inside the 32 as of K inside a k-group above, applied to T to match).
// blocks (otherwise): one CTA per 16-row block, eight warps splitting the
//   k-groups, four k-groups' loads in flight per warp straight into
//   registers, then the U rows and T from global memory.
//
// bf16 ring (ring_kernel<true, KU>): the same persistent ring with stages of
//   16 rows x KU 32-column groups of bf16 W0 (KU = 48 for up to two tokens,
//   32 above: 3 or 2 KB of each row per stage, as many 16-row x 1 KB TMA
//   boxes).  Longer runs of each row per request stream faster (Gemma-4
//   gate/up, M = 1: 1 KB 119.8 us, 2 KB 102.7, 3 KB 88.7).  Lane q's eight
//   consecutive columns of a 32-column group are the logical columns 2q,
//   2q + 1, 2q + 8, 2q + 9 of two MMAs, and the prep launch writes x in the
//   same order: [K/32][token][4][8] bf16.
#include <cuda_fp16.h>

#include <algorithm>
#include <atomic>

#include "wl_common.cuh"
#include "wl_internal.h"

namespace wl {

namespace {

constexpr int FW = 8;             // warps per CTA (consumer warps in the ring variant)
constexpr int FTH = 32 * FW;
constexpr int FKG = kFp4KGroup;   // 128 columns per k-group
constexpr int kPrepThreads = 256;
constexpr int kRingThreads = FTH + 32;  // + the producer warp
constexpr int kIssueLanes = 2;          // producer lanes issuing copies
constexpr uint32_t kCodeBytes = 16 * 64 * kFp4StageKG;   // 16 KB: 16 rows x 1024 bytes
constexpr uint32_t kTOff = 8192;  // U unit: T (M x r fp32) after U (16 x 2r bytes <= 8 KB)
constexpr uint32_t kRingSmemMax = 227 * 1024;
constexpr int kFp4RingMinK = 8192;         // NVFP4 calls with K at least this take the ring
constexpr int kFp4RingMinBlocks = 2048;    // ... and so do calls of at least this many 16-row blocks

__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7},"
        " {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7},"
        " {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint16_t lds16(uint32_t addr) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void consumer_bar() { asm volatile("bar.sync 1, %0;" ::"n"(FTH) : "memory"); }

__device__ __forceinline__ uint64_t evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ void tma_1d(void *dst, const void *tmap, int c0, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.1d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2}], [%3];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void tma_2d(void *dst, const void *tmap, int c0, int c1, uint64_t *bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(smem_addr(bar)), "l"(pol)
        : "memory");
}

// The eight E2M1 codes of a 32-bit word as four f16 pairs: byte b holds
// elements 2b (low nibble) and 2b + 1 (high nibble).
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t (&h)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
}

// Two E4M3 bytes (low byte first) as an f16 pair.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t v) {
    uint32_t h;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(v));
    return h;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Both halves of an f16 pair set to its low (hi = false) or high half.
__device__ __forceinline__ uint32_t hdup(uint32_t v, bool hi) {
    const uint32_t h = hi ? (v >> 16) : (v & 0xFFFFu);
    return h | (h << 16);
}

// One k-group of a lane: codes of rows g and g + 8 (16 bytes each), their
// scale byte pairs, and the lane's 32 x values per token (four 16-byte
// pieces); eight MMAs into four accumulators (MMA i into acc[i % 4]: short
// dependency chains).
__device__ __forceinline__ void kgroup_mma(float (&acc)[4][4], const uint4 &c0, const uint4 &c1, uint16_t s0,
                                           uint16_t s1, const uint4 (&xf)[4]) {
    const uint32_t xw[16] = {xf[0].x, xf[0].y, xf[0].z, xf[0].w, xf[1].x, xf[1].y, xf[1].z, xf[1].w,
                             xf[2].x, xf[2].y, xf[2].z, xf[2].w, xf[3].x, xf[3].y, xf[3].z, xf[3].w};
    const uint32_t sc0 = e4m3x2_to_f16x2(s0), sc1 = e4m3x2_to_f16x2(s1);
    const uint32_t cw0[4] = {c0.x, c0.y, c0.z, c0.w};
    const uint32_t cw1[4] = {c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
        // elements 8 wi .. 8 wi + 7 of the lane's 32: block scale 0 for the
        // first 16, 1 for the last 16
        uint32_t h0[4], h1[4];
        e2m1x8_to_f16x2(cw0[wi], h0);
        e2m1x8_to_f16x2(cw1[wi], h1);
        const uint32_t f0 = hdup(sc0, wi >= 2), f1 = hdup(sc1, wi >= 2);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            h0[e] = hmul2(h0[e], f0);
            h1[e] = hmul2(h1[e], f1);
        }
        // MMAs 2 wi and 2 wi + 1: elements 4i .. 4i + 3
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const uint32_t a[4] = {h0[2 * hh], h1[2 * hh], h0[2 * hh + 1], h1[2 * hh + 1]};
            mma_f16(acc[(2 * wi + hh) & 3], a, xw[4 * wi + 2 * hh], xw[4 * wi + 2 * hh + 1]);
        }
    }
}

// Index of x[m][k] in the permuted f16 copy.
__device__ __forceinline__ size_t xq_index(int m, int k, int Mp) {
    const int kg = k >> 7, c = k & 127, q = c >> 5, t = (c >> 3) & 3, j = c & 7;
    return ((((size_t)kg * 4 + t) * Mp + m) * 4 + q) * 8 + j;
}

// Index of x[m][k] in the permuted bf16 copy of the bf16-weight ring: per
// 32-column group, lane q's eight consecutive columns 8q .. 8q + 7, tokens
// (Mp of them) in between: [k / 32][m][q][8].
__device__ __forceinline__ size_t xb_index(int m, int k, int Mp) {
    return ((((size_t)(k >> 5) * Mp + m) * 4 + ((k >> 3) & 3)) * 8) + (k & 7);
}

// The pj-th projection with a delta (-1 if none).
__device__ __forceinline__ int delta_seg(const Fp4Params &P, int pj) {
    for (int i = 0, n = 0; i < P.nseg; ++i)
        if (P.seg[i].r > 0 && n++ == pj) return i;
    return -1;
}

}  // namespace

// ------------------------------------------------------------------ prep ---
// CTA (projection slot pj, slice sl): rows [sl * kr, ..) of V for the pj-th
// projection with a delta; CTAs of slot 0 also write their columns of x to
// the permuted f16 copy.
__global__ void __launch_bounds__(kPrepThreads) fp4_prep_kernel(const __grid_constant__ Fp4Params P) {
    pdl_launch_dependents();
    pdl_wait_primary();  // x is the previous kernel's output
    __shared__ float xs[kFp4MaxM * kFp4PrepMaxRows];
    __shared__ float red[2048];
    __shared__ int last;
    const int tid = threadIdx.x;
    const int S = P.slices, kr = P.kr;
    const int pj = blockIdx.x / S, sl = blockIdx.x - pj * S;
    const int K = P.K, M = P.M, Mp = P.Mp;
    const int k0 = sl * kr, k1 = min(K, k0 + kr), nk = k1 - k0;
    for (int i = tid; i < Mp * nk; i += kPrepThreads) {
        const int m = i / nk, k = k0 + i - m * nk;
        const __nv_bfloat16 xb = m < M ? P.x[(size_t)m * K + k] : __float2bfloat16_rn(0.f);
        const float v = __bfloat162float(xb);
        if (m < M) xs[m * kr + (k - k0)] = v;
        if (pj == 0) {
            if (P.bf16)
                reinterpret_cast<__nv_bfloat16 *>(P.xq)[xb_index(m, k, Mp)] = xb;
            else
                P.xq[xq_index(m, k, Mp)] = __float2half_rn(v);
        }
    }
    if (P.bf16 && pj == 0 && k1 == K) {
        // the last 32-column group's columns past K are zero
        const int kp = (K + 31) & ~31;
        for (int i = tid; i < Mp * (kp - K); i += kPrepThreads) {
            const int m = i / (kp - K), k = K + i - m * (kp - K);
            reinterpret_cast<__nv_bfloat16 *>(P.xq)[xb_index(m, k, Mp)] = __float2bfloat16_rn(0.f);
        }
    }
    __syncthreads();
    const int sp = delta_seg(P, pj);
    if (sp < 0) return;
    const Fp4Seg &sg = P.seg[sp];
    const int r = sg.r, t_ld = P.t_ld, t_off = sg.t_off;
    // threads: cgp (a power of two >= r / 8) 8-column groups x rs row lanes
    const int cg = r >> 3;
    int cgp = 1;
    while (cgp < cg) cgp <<= 1;
    const int rs = kPrepThreads / cgp, cgi = tid & (cgp - 1), rsub = tid / cgp;
    float acc[8][kFp4MaxM];
#pragma unroll
    for (int e = 0; e < 8; ++e)
#pragma unroll
        for (int m = 0; m < kFp4MaxM; ++m) acc[e][m] = 0.f;
    if (cgi < cg) {
        const uint4 *vp = reinterpret_cast<const uint4 *>(sg.V) + cgi;
        const int ld = r >> 3;  // uint4 per row of V
        // rows k0 + rsub, + rs, ...: four loads in flight, sums in row order
        for (int k = k0 + rsub; k < k1; k += 4 * rs) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int kk = k + u * rs;
                v[u] = kk < k1 ? __ldg(vp + (size_t)kk * ld) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int kk = k + u * rs;
                if (kk >= k1) break;
                const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int m = 0; m < kFp4MaxM; ++m) {
                    if (m >= M) break;
                    const float xv = xs[m * kr + (kk - k0)];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        acc[2 * e][m] = fmaf(bf16lo(w[e]), xv, acc[2 * e][m]);
                        acc[2 * e + 1][m] = fmaf(bf16hi(w[e]), xv, acc[2 * e + 1][m]);
                    }
                }
            }
        }
    }
    // the row lanes' sums, added in row-lane order, one token at a time
    for (int m = 0; m < M; ++m) {
        if (cgi < cg) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float a = acc[e][0];
#pragma unroll
                for (int mm = 1; mm < kFp4MaxM; ++mm)
                    if (mm == m) a = acc[e][mm];
                red[rsub * r + 8 * cgi + e] = a;
            }
        }
        __syncthreads();
        for (int j = tid; j < r; j += kPrepThreads) {
            float t = 0.f;
            for (int q = 0; q < rs; ++q) t += red[q * r + j];
            P.Tpart[((size_t)sl * M + m) * t_ld + t_off + j] = t;
        }
        __syncthreads();
    }
    // level 1: the last CTA of this group of slices adds the group's partials
    const int grp = sl / kFp4GroupSlices, g0 = grp * kFp4GroupSlices, gs = min(kFp4GroupSlices, S - g0);
    __threadfence();
    __syncthreads();
    if (tid == 0) last = atomicAdd(&P.cnt[pj * P.ngrp + grp], 1u) == (unsigned)(gs - 1);
    __syncthreads();
    if (!last) return;
    __threadfence();
    for (int i = tid; i < M * r; i += kPrepThreads) {
        const int m = i / r, j = i - m * r;
        float v[kFp4GroupSlices];
#pragma unroll
        for (int u = 0; u < kFp4GroupSlices; ++u)
            v[u] = u < gs ? __ldcg(P.Tpart + ((size_t)(g0 + u) * M + m) * t_ld + t_off + j) : 0.f;
        float t = 0.f;
#pragma unroll
        for (int u = 0; u < kFp4GroupSlices; ++u) t += v[u];  // slice order
        P.Gpart[((size_t)grp * M + m) * t_ld + t_off + j] = t;
    }
    if (tid == 0) P.cnt[pj * P.ngrp + grp] = 0u;  // for the next call
    // level 2: the last group adds the group sums in group order
    __threadfence();
    __syncthreads();
    unsigned int *pc = P.cnt + (size_t)P.nr * P.ngrp + pj;
    if (tid == 0) last = atomicAdd(pc, 1u) == (unsigned)(P.ngrp - 1);
    __syncthreads();
    if (!last) return;
    __threadfence();
    const int ng = P.ngrp;
    for (int i = tid; i < M * r; i += kPrepThreads) {
        const int m = i / r, j = i - m * r;
        float t = 0.f;
        for (int gb = 0; gb < ng; gb += 16) {
            float v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u)
                v[u] = gb + u < ng ? __ldcg(P.Gpart + ((size_t)(gb + u) * M + m) * t_ld + t_off + j) : 0.f;
#pragma unroll
            for (int u = 0; u < 16; ++u) t += v[u];
        }
        P.T[(size_t)m * t_ld + t_off + j] = t;
    }
    if (tid == 0) *pc = 0u;
}

// ---------------------------------------------------------- block stream ---
__global__ void __launch_bounds__(FTH, 2) fp4_block_kernel(const __grid_constant__ Fp4Params P) {
    pdl_launch_dependents();
    __shared__ float4 red[FW][32][2];  // each warp's fragments: W0 x, U T
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
    const int b = blockIdx.x;
    int sp = 0;
    while (sp + 1 < P.nseg && b >= P.seg[sp + 1].blk_begin) ++sp;
    const Fp4Seg &S = P.seg[sp];
    const int row0 = (b - S.blk_begin) * 16;
    const int K = P.K, M = P.M, N = S.N, Mp = P.Mp;
    const int nkg = K / FKG;
    const bool ok0 = row0 + g < N, ok1 = row0 + g + 8 < N;
    const uint8_t *cr0 = S.codes + (size_t)(ok0 ? row0 + g : row0) * (K / 2) + 16 * q;
    const uint8_t *cr1 = S.codes + (size_t)(ok1 ? row0 + g + 8 : row0) * (K / 2) + 16 * q;
    const uint8_t *sr0 = S.scales + (size_t)(ok0 ? row0 + g : row0) * (K / 16) + 2 * q;
    const uint8_t *sr1 = S.scales + (size_t)(ok1 ? row0 + g + 8 : row0) * (K / 16) + 2 * q;

    // The warp's k-groups (kg = warp, warp + 8, ...) FKB at a time: every
    // load of a batch -- codes and scale bytes, weights, so the first batch is
    // requested before the wait for the prep kernel -- is in flight before
    // the first is used.
    constexpr int FKB = 4;
    uint4 cb0[FKB], cb1[FKB];
    uint16_t sb0[FKB], sb1[FKB];
    auto load = [&](int kg0) {
#pragma unroll
        for (int i = 0; i < FKB; ++i) {
            const int k = kg0 + i * FW;
            const bool kv = k < nkg;
            cb0[i] = (kv && ok0) ? __ldg(reinterpret_cast<const uint4 *>(cr0 + (size_t)k * (FKG / 2)))
                                 : make_uint4(0u, 0u, 0u, 0u);
            cb1[i] = (kv && ok1) ? __ldg(reinterpret_cast<const uint4 *>(cr1 + (size_t)k * (FKG / 2)))
                                 : make_uint4(0u, 0u, 0u, 0u);
            sb0[i] = (kv && ok0) ? __ldg(reinterpret_cast<const unsigned short *>(sr0 + (size_t)k * (FKG / 16)))
                                 : (uint16_t)0;
            sb1[i] = (kv && ok1) ? __ldg(reinterpret_cast<const unsigned short *>(sr1 + (size_t)k * (FKG / 16)))
                                 : (uint16_t)0;
        }
    };
    load(warp);
    // the U rows of this warp's first 32 rank columns are weights too
    const int r = S.r;
    const int ju = warp * 32 + 8 * q;  // this lane's eight rank columns of group jg = warp
    const bool juv = ju < r;
    const uint4 ulo0 = (juv && ok0) ? __ldg(reinterpret_cast<const uint4 *>(S.U + (size_t)(row0 + g) * r + ju))
                                    : make_uint4(0u, 0u, 0u, 0u);
    const uint4 uhi0 = (juv && ok1) ? __ldg(reinterpret_cast<const uint4 *>(S.U + (size_t)(row0 + g + 8) * r + ju))
                                    : make_uint4(0u, 0u, 0u, 0u);
    pdl_wait_primary();  // xq and T are the prep kernel's
    const bool xv = g < M;
    float tu0[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) tu0[e] = (juv && xv) ? __ldcg(P.T + (size_t)g * P.t_ld + S.t_off + ju + e) : 0.f;

    float acc[4][4] = {};
    for (int kg0 = warp; kg0 < nkg; kg0 += FW * FKB) {
        if (kg0 != warp) load(kg0);
#pragma unroll
        for (int i = 0; i < FKB; ++i) {
            const int kg = kg0 + i * FW;
            if (kg >= nkg) break;
            uint4 xf[4];
#pragma unroll
            for (int t = 0; t < 4; ++t)
                xf[t] = xv ? __ldg(reinterpret_cast<const uint4 *>(P.xq) + ((((size_t)kg * 4 + t) * Mp + g) * 4 + q))
                           : make_uint4(0u, 0u, 0u, 0u);
            kgroup_mma(acc, cb0[i], cb1[i], sb0[i], sb1[i], xf);
        }
    }

    // ---- U T over 32-column groups of the rank ----
    float acd[4] = {0.f, 0.f, 0.f, 0.f};
    for (int jg = warp; jg * 32 < r; jg += FW) {
        const int j = jg * 32 + 8 * q;  // this lane's eight rank columns
        const bool jv = j < r, first = jg == warp;
        const uint4 ulo = first ? ulo0
                                : (jv && ok0) ? __ldg(reinterpret_cast<const uint4 *>(S.U + (size_t)(row0 + g) * r + j))
                                              : make_uint4(0u, 0u, 0u, 0u);
        const uint4 uhi = first ? uhi0
                                : (jv && ok1) ? __ldg(reinterpret_cast<const uint4 *>(S.U + (size_t)(row0 + g + 8) * r + j))
                                              : make_uint4(0u, 0u, 0u, 0u);
        float t[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
            t[e] = first ? tu0[e] : (jv && xv) ? __ldcg(P.T + (size_t)g * P.t_ld + S.t_off + j + e) : 0.f;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const uint32_t a[4] = {hh ? ulo.z : ulo.x, hh ? uhi.z : uhi.x, hh ? ulo.w : ulo.y, hh ? uhi.w : uhi.y};
            const uint32_t b0 = pack_bf16x2(t[4 * hh], t[4 * hh + 1]), b1 = pack_bf16x2(t[4 * hh + 2], t[4 * hh + 3]);
            const uint32_t l0 = pack_bf16x2(t[4 * hh] - bf16lo(b0), t[4 * hh + 1] - bf16hi(b0));
            const uint32_t l1 = pack_bf16x2(t[4 * hh + 2] - bf16lo(b1), t[4 * hh + 3] - bf16hi(b1));
            mma_bf16(acd, a, b0, b1);
            mma_bf16(acd, a, l0, l1);
        }
    }
    red[warp][lane][0] = make_float4((acc[0][0] + acc[1][0]) + (acc[2][0] + acc[3][0]),
                                     (acc[0][1] + acc[1][1]) + (acc[2][1] + acc[3][1]),
                                     (acc[0][2] + acc[1][2]) + (acc[2][2] + acc[3][2]),
                                     (acc[0][3] + acc[1][3]) + (acc[2][3] + acc[3][3]));
    red[warp][lane][1] = make_float4(acd[0], acd[1], acd[2], acd[3]);
    __syncthreads();
    // output (row rr, token m): fragment lane (rr & 7) * 4 + (m >> 1), element
    // (rr >> 3) * 2 + (m & 1); the eight warps' sums in warp order
    for (int e = tid; e < 16 * M; e += FTH) {
        const int rr = e / M, m = e - rr * M;
        if (row0 + rr >= N) continue;
        const int fl = (rr & 7) * 4 + (m >> 1), fe = (rr >> 3) * 2 + (m & 1);
        float z = 0.f, d = 0.f;
#pragma unroll
        for (int w = 0; w < FW; ++w) {
            z += reinterpret_cast<const float *>(&red[w][fl][0])[fe];
            d += reinterpret_cast<const float *>(&red[w][fl][1])[fe];
        }
        const float sc = __ldg(S.s + row0 + rr) * S.ts;
        S.y[(size_t)m * N + row0 + rr] = __float2bfloat16_rn(fmaf(sc, z, d));
    }
}

// ----------------------------------------------------------- ring stream ---
namespace {

// Walks the units of the call in order: projection, block, stage.
struct UnitCursor {
    int sp, blk, st;
    __device__ void seek(const Fp4Params &P, long long u) {
        sp = 0;
        while (sp + 1 < P.nseg && u >= P.seg[sp + 1].ub) ++sp;
        const long long l = u - P.seg[sp].ub;
        blk = (int)(l / P.seg[sp].upb);
        st = (int)(l - (long long)blk * P.seg[sp].upb);
    }
    __device__ void next(const Fp4Params &P) {
        if (sp >= P.nseg) return;  // past the last unit
        if (++st == P.seg[sp].upb) {
            st = 0;
            if (++blk * 16 >= P.seg[sp].N) {
                blk = 0;
                ++sp;
            }
        }
    }
};

__device__ __forceinline__ long long range_start(long long utot, int G, int c) {
    return (long long)(((unsigned long long)utot * (unsigned long long)c) / (unsigned long long)G);
}

// The CTA whose range holds unit u.
__device__ __forceinline__ int cta_of(long long utot, int G, long long u) {
    return (int)((((unsigned long long)u + 1ull) * (unsigned long long)G - 1ull) / (unsigned long long)utot);
}

}  // namespace

template <bool BF16, int KU>
__global__ void __launch_bounds__(kRingThreads, 1) ring_kernel(const __grid_constant__ Fp4Params P) {
    pdl_launch_dependents();
    extern __shared__ uint8_t dyn_smem[];
    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
    const int NS = P.ns;
    const uint32_t SB = (uint32_t)P.slot_bytes;
    float4 *red = reinterpret_cast<float4 *>(ring + (size_t)NS * SB);  // [2][FW][32][2]
    uint64_t *full = reinterpret_cast<uint64_t *>(red + 2 * FW * 32 * 2);
    uint64_t *empty = full + NS;
    // flags: [0] abort, [1] finisher of a split block, [2 + l] issue lane l's first unit not issued
    volatile int *flags = reinterpret_cast<volatile int *>(empty + NS);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x, c = blockIdx.x;
    const long long utot = P.utot;
    const long long u0 = range_start(utot, G, c), u1 = range_start(utot, G, c + 1);
    // k-units: 128-column k-groups of NVFP4 codes (KU = 16 per stage: 1 KB
    // of each row, one TMA box), or 32-column groups of bf16 weights (KU =
    // 48 or 32 per stage: 3 or 2 KB of each row, as many boxes).  Long runs
    // of each row per request stream faster (measured on the Gemma-4 gate/up
    // call at M = 1: 1 KB 119.8 us, 2 KB 102.7, 3 KB 90.5, 4 KB 92.6).
    static_assert(KU % FW == 0 && KU % kFp4StageKG == 0, "k-units of a stage");
    constexpr uint32_t WB = 16u * 64u * KU;            // weight bytes of a stage
    constexpr int NBOX = (int)(WB / kCodeBytes);       // 16-row x 1 KB boxes per stage
    constexpr uint32_t SCB = BF16 ? 0u : 16u * 8u * KU;  // block scales of a stage (8 bytes per row and k-group)
    const int K = P.K, M = P.M, Mp = P.Mp, nst = P.nst;
    const int nkg = BF16 ? (K + 31) / 32 : K / FKG;
    const uint32_t xstage = (BF16 ? 64u : 256u) * (uint32_t)Mp;  // bytes of permuted x per k-unit
    const uint32_t sv_off = WB + SCB + (uint32_t)KU * xstage;     // 16 row scales

    if (warp == FW && lane < P.nseg) {
        // the tensor maps into the descriptor cache before the first copy
        prefetch_tmap(&P.tm_c[lane]);
        if (!BF16) prefetch_tmap(&P.tm_s[lane]);
        prefetch_tmap(&P.tm_sv[lane]);
        if (P.seg[lane].r > 0) prefetch_tmap(&P.tm_u[lane]);
    }
    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], FW);
        }
        for (int k = 0; k < 2 + kIssueLanes; ++k) flags[k] = 0;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == FW) {
        // ---------------- producer ----------------
        // kIssueLanes lanes issue the copies, lane l those of units
        // i = l, l + kIssueLanes, ...: one thread alone could not issue them
        // fast enough to keep the ring full.
        if (lane < kIssueLanes) {
            const uint64_t pol = evict_first_policy();
            // 32-bit counters kept incrementally: a 64-bit division per unit
            // would cost more than the copies' issue
            const int n = (int)(u1 - u0), nfill = n < NS ? n : NS;
            UnitCursor cu;
            cu.seek(P, u0 + lane);
            int i = lane, slot = lane, round = 0;  // slot = i % NS, round = i / NS (NS >= kIssueLanes)
            bool waited = false;
            // the prep kernel's outputs a unit needs: the stage's x slice, or
            // (U unit) this projection's T, one row per token
            auto issue_dep = [&](int sl, const UnitCursor &c) {
                if (c.st < nst) {
                    const int kgs = min(KU, nkg - KU * c.st);
                    bulk_load(ring + (size_t)sl * SB + WB + SCB,
                              reinterpret_cast<const uint8_t *>(P.xq) + (size_t)KU * c.st * xstage,
                              (uint32_t)kgs * xstage, &full[sl]);
                } else {
                    const Fp4Seg &S2 = P.seg[c.sp];
                    for (int m = 0; m < M; ++m)
                        bulk_load(ring + (size_t)sl * SB + kTOff + (size_t)m * S2.r * 4, P.T + (size_t)m * P.t_ld + S2.t_off,
                                  (uint32_t)S2.r * 4u, &full[sl]);
                }
            };
            auto wait_primary = [&]() {
                // the weight tiles of this lane's units among the first NS are
                // requested; the x slices are the prep kernel's output
                pdl_wait_primary();
                waited = true;
                UnitCursor cw;
                cw.seek(P, u0 + lane);
                for (int ii = lane; ii < nfill; ii += kIssueLanes) {  // slot ii
                    issue_dep(ii, cw);
                    for (int k = 0; k < kIssueLanes; ++k) cw.next(P);
                }
            };
            for (; i < n; i += kIssueLanes) {
                if (!waited && i >= NS) wait_primary();
                uint8_t *sb = ring + (size_t)slot * SB;
                if (i >= NS &&
                    (flags[0] || !mbar_wait(&empty[slot], (uint32_t)(round - 1) & 1u, P.status, P.timeout_ns))) {
                    flags[0] = 1;
                    break;
                }
                const Fp4Seg &S = P.seg[cu.sp];
                const int row0 = cu.blk * 16;
                // the block's first unit in this CTA's range also brings its 16 row scales
                const bool first = i == 0 || cu.st == 0;
                const uint32_t sbytes = first ? 64u : 0u;
                if (cu.st < nst) {
                    const int kgs = min(KU, nkg - KU * cu.st);
                    mbar_arrive_expect_tx(&full[slot], WB + SCB + (uint32_t)kgs * xstage + sbytes);
#pragma unroll
                    for (int bx = 0; bx < NBOX; ++bx)
                        tma_2d(sb + (size_t)bx * kCodeBytes, &P.tm_c[cu.sp], (int)(kCodeBytes / 64) * (NBOX * cu.st + bx),
                               row0, &full[slot], pol);
                    if (!BF16)
                        tma_2d(sb + WB, &P.tm_s[cu.sp], 2 * KU * cu.st, row0, &full[slot], pol);
                } else {
                    mbar_arrive_expect_tx(&full[slot], 32u * (uint32_t)S.r + 4u * (uint32_t)(M * S.r) + sbytes);
                    tma_2d(sb, &P.tm_u[cu.sp], 0, row0, &full[slot], pol);
                }
                if (first) tma_1d(sb + sv_off, &P.tm_sv[cu.sp], row0, &full[slot]);
                if (waited) issue_dep(slot, cu);
                for (int k = 0; k < kIssueLanes; ++k) cu.next(P);
                if ((slot += kIssueLanes) >= NS) {
                    slot -= NS;
                    ++round;
                }
            }
            flags[2 + lane] = i;  // this lane's first unit not issued
            if (!waited) wait_primary();
        }
    } else {
        // ---------------- consumers ----------------
        pdl_wait_primary();  // T is the prep kernel's output
        const int g = lane >> 2, q = lane & 3;
        const bool xv = g < M;
        float acc[4][4] = {};
        float acd[4] = {0.f, 0.f, 0.f, 0.f};
        int par = 0;
        const uint32_t ring_a = smem_addr(ring);
        UnitCursor cu;
        cu.seek(P, u0);
        int nslot = 0;
        uint32_t nphase = 0;
        // output e = (row rr, token m) = lane * 8 + warp of a block: the
        // epilogue's work spread over all warps
        const int eo = lane * FW + warp;
        float sv = 0.f;
        for (long long u = u0; u < u1; ++u) {
            const int slot = nslot;
            const uint32_t phase = nphase;
            if (++nslot == NS) {
                nslot = 0;
                nphase ^= 1u;
            }
            const uint32_t sa = ring_a + (uint32_t)slot * SB;
            const Fp4Seg &S = P.seg[cu.sp];
            const bool ok = !flags[0] && mbar_wait(&full[slot], phase, P.status, P.timeout_ns);
            if (!ok) flags[0] = 1;
            if (ok && (u == u0 || cu.st == 0) && eo < 16 * M)  // a new block: this thread's row scale
                sv = __uint_as_float(lds32(sa + sv_off + 4u * (uint32_t)(eo / M))) * S.ts;
            if (ok) {
                if (cu.st < nst) {
                    // k-groups warp and warp + 8 of the stage; codes: row g at
                    // 1024 g; scales: row g at 128 g
#pragma unroll
                    for (int j = 0; j < KU / FW; ++j) {
                        const int kgl = warp + FW * j;
                        if (KU * cu.st + kgl >= nkg) break;
                        // box kgl / 16, rows 1 KB apart inside it
                        const uint32_t cb = sa + (uint32_t)(kgl >> 4) * kCodeBytes + 64u * (kgl & 15) + 16u * q;
                        if (BF16) {
                            // 32 columns of rows g and g + 8: the lane's eight
                            // (8q .. 8q + 7) are the logical columns 2q, 2q + 1,
                            // 2q + 8, 2q + 9 of two MMAs, as in x's copy
                            const uint4 w0 = lds128(cb + g * (kCodeBytes / 16)), w1 = lds128(cb + (g + 8) * (kCodeBytes / 16));
                            const uint4 bx = xv ? lds128(sa + WB + (uint32_t)(((kgl * Mp + g) * 4 + q) * 16))
                                                : make_uint4(0u, 0u, 0u, 0u);
                            const uint32_t a1[4] = {w0.x, w1.x, w0.y, w1.y};
                            const uint32_t a2[4] = {w0.z, w1.z, w0.w, w1.w};
                            mma_bf16(acc[(2 * j) & 3], a1, bx.x, bx.y);
                            mma_bf16(acc[(2 * j + 1) & 3], a2, bx.z, bx.w);
                            continue;
                        }
                        const uint4 c0 = lds128(cb + g * (kCodeBytes / 16)), c1 = lds128(cb + (g + 8) * (kCodeBytes / 16));
                        const uint32_t sbs = sa + WB + 8u * kgl + 2u * q;
                        const uint16_t s0 = lds16(sbs + g * (SCB / 16)), s1 = lds16(sbs + (g + 8) * (SCB / 16));
                        uint4 xf[4];
                        const uint32_t xb = sa + WB + SCB;
#pragma unroll
                        for (int t = 0; t < 4; ++t)
                            xf[t] = xv ? lds128(xb + (uint32_t)((((kgl * 4 + t) * Mp + g) * 4 + q) * 16))
                                       : make_uint4(0u, 0u, 0u, 0u);
                        kgroup_mma(acc, c0, c1, s0, s1, xf);
                    }
                } else if (32 * warp < S.r) {  // warp-uniform: the MMAs below are collective
                    // T as bf16 high / low B fragments: token g, rank columns
                    // 32 warp + 8q .. + 7 (MMA hh: four of them)
                    const bool jv = 32 * warp + 8 * q < S.r;
                    const uint32_t ta = sa + kTOff + 4u * (uint32_t)(g * S.r + 32 * warp + 8 * q);
                    const uint4 t0 = (jv && xv) ? lds128(ta) : make_uint4(0u, 0u, 0u, 0u);
                    const uint4 t1 = (jv && xv) ? lds128(ta + 16u) : make_uint4(0u, 0u, 0u, 0u);
                    const float t[8] = {__uint_as_float(t0.x), __uint_as_float(t0.y), __uint_as_float(t0.z),
                                        __uint_as_float(t0.w), __uint_as_float(t1.x), __uint_as_float(t1.y),
                                        __uint_as_float(t1.z), __uint_as_float(t1.w)};
                    uint32_t tb[2][4];  // [MMA][b0, b1, low b0, low b1]
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const uint32_t h0 = pack_bf16x2(t[4 * hh], t[4 * hh + 1]);
                        const uint32_t h1 = pack_bf16x2(t[4 * hh + 2], t[4 * hh + 3]);
                        tb[hh][0] = h0;
                        tb[hh][1] = h1;
                        tb[hh][2] = pack_bf16x2(t[4 * hh] - bf16lo(h0), t[4 * hh + 1] - bf16hi(h0));
                        tb[hh][3] = pack_bf16x2(t[4 * hh + 2] - bf16lo(h1), t[4 * hh + 3] - bf16hi(h1));
                    }
                    // U rows g and g + 8 (2r bytes each): the lane's eight ranks
                    const uint32_t ub = sa + 64u * warp + 16u * q;
                    const uint4 ulo = jv ? lds128(ub + (uint32_t)g * 2u * S.r) : make_uint4(0u, 0u, 0u, 0u);
                    const uint4 uhi = jv ? lds128(ub + (uint32_t)(g + 8) * 2u * S.r) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const uint32_t a[4] = {hh ? ulo.z : ulo.x, hh ? uhi.z : uhi.x, hh ? ulo.w : ulo.y,
                                               hh ? uhi.w : uhi.y};
                        mma_bf16(acd, a, tb[hh][0], tb[hh][1]);
                        mma_bf16(acd, a, tb[hh][2], tb[hh][3]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
            const int blk = cu.blk, upb = S.upb;
            const bool block_end = cu.st == upb - 1 || u == u1 - 1;
            cu.next(P);
            if (!block_end) continue;

            // ---- the block's sums: warps in order ----
            float4 *rd = red + (size_t)par * FW * 32 * 2;
            rd[(warp * 32 + lane) * 2] = make_float4((acc[0][0] + acc[1][0]) + (acc[2][0] + acc[3][0]),
                                                     (acc[0][1] + acc[1][1]) + (acc[2][1] + acc[3][1]),
                                                     (acc[0][2] + acc[1][2]) + (acc[2][2] + acc[3][2]),
                                                     (acc[0][3] + acc[1][3]) + (acc[2][3] + acc[3][3]));
            rd[(warp * 32 + lane) * 2 + 1] = make_float4(acd[0], acd[1], acd[2], acd[3]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc[0][e] = acc[1][e] = acc[2][e] = acc[3][e] = 0.f;
                acd[e] = 0.f;
            }
            consumer_bar();
            const long long ub = S.ub + (long long)blk * upb, ue = ub + upb;
            const int row0 = blk * 16, N = S.N;
            const int e = eo;
            const int rr = e / M, m = e - rr * M;
            const bool has = e < 16 * M && row0 + rr < N;
            float z = 0.f, d = 0.f;
            if (e < 16 * M) {
                const int fl = (rr & 7) * 4 + (m >> 1), fe = (rr >> 3) * 2 + (m & 1);
#pragma unroll
                for (int w = 0; w < FW; ++w) {
                    z += reinterpret_cast<const float *>(&rd[(w * 32 + fl) * 2])[fe];
                    d += reinterpret_cast<const float *>(&rd[(w * 32 + fl) * 2 + 1])[fe];
                }
            }
            par ^= 1;
            if (ub >= u0 && ue <= u1) {
                if (has && !flags[0]) S.y[(size_t)m * N + row0 + rr] = __float2bfloat16_rn(fmaf(sv, z, d));
                continue;
            }
            // ---- a block split between CTAs: the last to arrive finishes it ----
            // slot 0: the block holding this CTA's first unit; slot 1: its last block
            const int mys = u0 >= ub ? 0 : 1;
            if (e < 16 * M) P.parts[((size_t)c * 2 + mys) * (16 * kFp4MaxM) + e] = make_float2(z, d);
            __threadfence();
            consumer_bar();
            const int cf = cta_of(utot, G, ub), cl = cta_of(utot, G, ue - 1);
            const int gb = S.blk_begin + blk;
            if (tid == 0) {
                const unsigned prev = atomicAdd(&P.bcnt[gb], 1u);
                flags[1] = prev == (unsigned)(cl - cf);
                if (prev == (unsigned)(cl - cf)) {
                    __threadfence();
                    P.bcnt[gb] = 0u;  // for the next call
                }
            }
            consumer_bar();
            if (flags[1] && has && !flags[0]) {
                float zs = 0.f, ds = 0.f;
                for (int cc = cf; cc <= cl; ++cc) {
                    const int s2 = range_start(utot, G, cc) >= ub ? 0 : 1;
                    const float2 pz = __ldcg(P.parts + ((size_t)cc * 2 + s2) * (16 * kFp4MaxM) + e);
                    zs += pz.x;
                    ds += pz.y;
                }
                S.y[(size_t)m * N + row0 + rr] = __float2bfloat16_rn(fmaf(sv, zs, ds));
            }
            consumer_bar();  // flags[1] is rewritten by the next split block
        }
    }
    __syncthreads();
    if (flags[0] && tid == 0) {
        // after a time-out: wait (bounded) for the last copies issued into
        // each slot before the CTA's shared memory is released (unit i was
        // issued iff i is below its lane's stop)
        const long long n = u1 - u0;
        for (int s = 0; s < NS && s < n; ++s) {
            long long last = -1;
            for (long long ii = s; ii < n; ii += NS)
                if (ii < flags[2 + (int)(ii % kIssueLanes)]) last = ii;
            if (last >= 0) mbar_wait(&full[s], (uint32_t)(last / NS) & 1u, nullptr, P.timeout_ns);
        }
    }
}

// ------------------------------------------------------------------ host ---
namespace {
std::atomic<bool> g_ring_attr{false};
}

size_t fp4_xq_halves(const Fp4Params &p) {
    return p.bf16 ? (size_t)((p.K + 31) / 32) * 32 * p.Mp : (size_t)(p.K / FKG) * 4 * p.Mp * 4 * 8;
}

wl_status plan_fp4(Fp4Params &p, int num_sms, bool encode_maps) {
    const int K = p.K, M = p.M;
    p.Mp = M <= 1 ? 1 : (M + 1) & ~1;
    // prep: about two CTAs per SM over the projections with a delta
    const int nrr = p.nr > 0 ? p.nr : 1;
    const int target = (2 * num_sms + nrr - 1) / nrr;
    int kr = (K + target - 1) / target;
    kr = (kr + 7) / 8 * 8;
    if (p.nr == 0) kr = kFp4PrepMaxRows;
    kr = std::max(8, std::min(kr, kFp4PrepMaxRows));
    p.kr = kr;
    p.slices = (K + kr - 1) / kr;
    p.ngrp = (p.slices + kFp4GroupSlices - 1) / kFp4GroupSlices;
    // ring stream when every rank fits one U unit, s is 16-byte aligned (its
    // TMA box) and, for NVFP4, the scale rows are 16-byte strided
    bool ring = p.bf16 ? true : K % 256 == 0;
    for (int i = 0; i < p.nseg; ++i)
        ring = ring && p.seg[i].r <= kFp4RingMaxRank && (reinterpret_cast<uintptr_t>(p.seg[i].s) & 15u) == 0 &&
               (p.bf16 || (reinterpret_cast<uintptr_t>(p.seg[i].scales) & 15u) == 0);
    // NVFP4: and when K is long or the call has many row blocks; otherwise
    // one CTA per block streams faster (measured on the Gemma-4-31B families
    // at M = 1, rank 256, ring against block stream: gate/up 69.7 / 72.0 us,
    // down 35.6 / 41.0, o 5376 x 8192 24.3 / 26.2, but q 8192 x 5376 27.3 /
    // 24.5).  bf16 weights: the caller decides.
    if (!p.bf16) ring = ring && (K >= kFp4RingMinK || p.total_blocks >= kFp4RingMinBlocks);
    p.ring = ring ? 1 : 0;
    if (!ring) return p.bf16 ? WL_ERR_UNSUPPORTED : WL_OK;
    const int nkg = p.bf16 ? (K + 31) / 32 : K / FKG;  // k-units
    // per stage (the kernel's KU): bf16 rows of 3 KB per stage for up to two
    // token rows of x, of 2 KB above (the x slices grow with the tokens and
    // the ring must keep enough slots)
    const int ku = p.Mp <= 2 ? (p.bf16 ? 3 : 2) * kFp4StageKG : (p.bf16 ? 2 : 1) * kFp4StageKG;
    p.ku = ku;
    p.nst = (nkg + ku - 1) / ku;
    long long ub = 0;
    for (int i = 0; i < p.nseg; ++i) {
        Fp4Seg &sg = p.seg[i];
        sg.ub = ub;
        sg.upb = p.nst + (sg.r > 0 ? 1 : 0);
        ub += (long long)((sg.N + 15) / 16) * sg.upb;
    }
    p.utot = ub;
    p.grid = (int)std::min<long long>(num_sms, ub);
    const uint32_t slot = (16u * 64u * ku + (p.bf16 ? 0u : 16u * 8u * ku) + (uint32_t)ku * (p.bf16 ? 64u : 256u) * p.Mp +
                           64u + 1023u) &
                          ~1023u;
    p.slot_bytes = (int)slot;
    const uint32_t fixed = 2u * FW * 32 * 2 * 16 + 32 + 1024;  // reduction buffers, flags, alignment
    int ns = (int)((kRingSmemMax - fixed) / (slot + 16));
    ns = std::min(ns, kFp4RingMaxStages);
    if (ns < kIssueLanes) {
        p.ring = 0;
        return p.bf16 ? WL_ERR_UNSUPPORTED : WL_OK;
    }
    p.ns = ns;
    p.smem = (int)((uint32_t)ns * slot + 2u * FW * 32 * 2 * 16 + 16u * ns + 32 + 1024);
    for (int i = 0; encode_maps && i < p.nseg; ++i) {
        const Fp4Seg &sg = p.seg[i];
        wl_status st;
        // the weight rows as 32-bit words (K/8 of them for NVFP4 codes, K/2 for bf16)
        const uint64_t wwords = p.bf16 ? (uint64_t)K / 2 : (uint64_t)K / 8;
        if ((st = encode_map_2d_u32(&p.tm_c[i], sg.codes, wwords, sg.N, wwords * 4, kCodeBytes / 64, 16)) != WL_OK)
            return st;
        if (!p.bf16 &&
            (st = encode_map_2d_u32(&p.tm_s[i], sg.scales, (uint64_t)K / 64, sg.N, (uint64_t)K / 16, 2u * ku, 16)) !=
                WL_OK)
            return st;
        if (sg.r > 0 &&
            (st = encode_map_2d_u32(&p.tm_u[i], sg.U, (uint64_t)sg.r / 2, sg.N, (uint64_t)sg.r * 2, sg.r / 2, 16)) !=
                WL_OK)
            return st;
        if ((st = encode_map_1d_f32(&p.tm_sv[i], sg.s, sg.N, 16)) != WL_OK) return st;
    }
    return WL_OK;
}

cudaError_t launch_fp4(const Fp4Params &p, cudaStream_t stream) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kPrepThreads);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3((unsigned)(p.slices * (p.nr > 0 ? p.nr : 1)));
    cudaError_t e = cudaLaunchKernelEx(&cfg, fp4_prep_kernel, p);
    if (e != cudaSuccess) return e;
    if (p.ring) {
        if (!g_ring_attr.load(std::memory_order_acquire)) {
            e = cudaFuncSetAttribute(ring_kernel<false, kFp4StageKG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kRingSmemMax);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(ring_kernel<false, 2 * kFp4StageKG>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRingSmemMax);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(ring_kernel<true, 2 * kFp4StageKG>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRingSmemMax);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(ring_kernel<true, 3 * kFp4StageKG>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRingSmemMax);
            if (e != cudaSuccess) return e;
            g_ring_attr.store(true, std::memory_order_release);
        }
        cfg.blockDim = dim3(kRingThreads);
        cfg.gridDim = dim3((unsigned)p.grid);
        cfg.dynamicSmemBytes = (size_t)p.smem;
        if (!p.bf16)
            return p.ku == 2 * kFp4StageKG ? cudaLaunchKernelEx(&cfg, ring_kernel<false, 2 * kFp4StageKG>, p)
                                           : cudaLaunchKernelEx(&cfg, ring_kernel<false, kFp4StageKG>, p);
        return p.ku == 3 * kFp4StageKG ? cudaLaunchKernelEx(&cfg, ring_kernel<true, 3 * kFp4StageKG>, p)
                                       : cudaLaunchKernelEx(&cfg, ring_kernel<true, 2 * kFp4StageKG>, p);
    }
    cfg.blockDim = dim3(FTH);
    cfg.gridDim = dim3((unsigned)p.total_blocks);
    return cudaLaunchKernelEx(&cfg, fp4_block_kernel, p);
}

}  // namespace wl
