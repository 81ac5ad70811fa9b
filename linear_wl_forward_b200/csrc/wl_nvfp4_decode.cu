// Decode with an NVFP4 shared block: y = s (.) (W0 x) + U (V^T x) where W0 is
// stored as FP4 E2M1 codes (two per byte, element 2i in the low nibble of
// byte i), one FP8 E4M3 scale per 16 consecutive elements of a row, and one
// fp32 tensor scale -- 0.5625 bytes per element instead of 2 ("Compression",
// "NVFP4: 3.18x smaller weights": packed 4-bit weights with an e4m3 scale per
// 16 elements, dequantised on the fly).  U, V and s stay as in the bf16 path.
//
// Two launches per call:
//  * prep: T = V^T x (fp32) for every projection with a delta, over slices
//    of K (one CTA per slice and projection, each thread one rank column,
//    fp32 sums in row order); the last CTA to finish a projection's slices
//    adds them up in slice order (no float atomics).  The same launch writes
//    x as f16 for the stream kernel.
//  * stream: one CTA per 16-row block of W0.  Its eight warps split the
//    128-column k-groups of K (four k-groups' loads in flight per warp); per
//    k-group each lane loads 16 bytes of codes
//    of row g and of row g + 8 (32 elements each, columns 32q .. 32q + 31 of
//    the k-group) and their two scale bytes straight into registers, expands
//    them with the hardware E2M1 -> f16 and E4M3 -> f16 conversions and one
//    f16 multiply per pair (an E2M1 value times an E4M3 scale is exact in
//    f16), and runs eight m16n8k16 MMAs (f16 in, fp32 accumulate): MMA i takes
//    the lane's elements 4i .. 4i + 3 as its logical columns 2q, 2q + 1,
//    2q + 8, 2q + 9 -- a fixed permutation of K inside the k-group, applied to
//    x identically.  The warps then multiply the U rows of the block by T (bf16
//    high and low parts of T, two MMAs) over 32-column groups of the rank, the
//    partial sums are added in warp order, and
//        y = bf16_rn((s * tensor_scale) * z + U T).
// The tensor scale multiplies s (both are per-row factors of the W0 product).
#include <cuda_fp16.h>

#include "wl_common.cuh"
#include "wl_internal.h"

namespace wl {

namespace {

constexpr int FW = 8;             // warps per CTA
constexpr int FTH = 32 * FW;
constexpr int FKG = kFp4KGroup;   // 128 columns per k-group
constexpr int kPrepRows = 64;     // K rows of V per prep CTA

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

}  // namespace

// ------------------------------------------------------------------ prep ---
// CTA (projection slot pj, slice sl): rows [sl * kPrepRows, ..) of V for the
// pj-th projection with a delta; CTAs of slot 0 also convert their columns of
// x to f16.
__global__ void __launch_bounds__(FTH) fp4_prep_kernel(const __grid_constant__ Fp4Params P) {
    pdl_launch_dependents();
    pdl_wait_primary();  // x is the previous kernel's output
    __shared__ float xs[kFp4MaxM * kPrepRows];
    __shared__ int last;
    const int S = P.slices;
    const int pj = blockIdx.x / S, sl = blockIdx.x - pj * S;
    const int K = P.K, M = P.M;
    const int k0 = sl * kPrepRows, k1 = min(K, k0 + kPrepRows);
    for (int i = threadIdx.x; i < M * (k1 - k0); i += FTH) {
        const int m = i / (k1 - k0), k = k0 + i - m * (k1 - k0);
        const float v = __bfloat162float(P.x[(size_t)m * K + k]);
        xs[m * kPrepRows + (k - k0)] = v;
        if (pj == 0) P.xh[(size_t)m * K + k] = __float2half_rn(v);
    }
    __syncthreads();
    // the pj-th projection with a delta
    int sp = -1;
    for (int i = 0, n = 0; i < P.nseg; ++i)
        if (P.seg[i].r > 0 && n++ == pj) sp = i;
    if (sp < 0) return;
    const Fp4Seg &sg = P.seg[sp];
    const int r = sg.r;
    float *part = P.Tpart + (size_t)S * M * sg.t_off;  // [S][M][r] of this projection
    for (int j = threadIdx.x; j < r; j += FTH) {
        float acc[kFp4MaxM];
#pragma unroll
        for (int m = 0; m < kFp4MaxM; ++m) acc[m] = 0.f;
        // 32 rows of V at a time: their loads are all in flight before the
        // first is used (sums stay in row order)
        for (int kb = k0; kb < k1; kb += 32) {
            float v[32];
#pragma unroll
            for (int u = 0; u < 32; ++u)
                v[u] = kb + u < k1 ? __bfloat162float(sg.V[(size_t)(kb + u) * r + j]) : 0.f;
#pragma unroll
            for (int u = 0; u < 32; ++u)
#pragma unroll
                for (int m = 0; m < kFp4MaxM; ++m)
                    if (m < M && kb + u < k1) acc[m] = fmaf(v[u], xs[m * kPrepRows + (kb + u - k0)], acc[m]);
        }
#pragma unroll
        for (int m = 0; m < kFp4MaxM; ++m)
            if (m < M) part[((size_t)sl * M + m) * r + j] = acc[m];
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(&P.cnt[pj], 1u) == (unsigned)(S - 1);
    __syncthreads();
    if (!last) return;
    __threadfence();
    for (int i = threadIdx.x; i < M * r; i += FTH) {
        const int m = i / r, j = i - m * r;
        float t = 0.f;
        for (int sb = 0; sb < S; sb += 32) {  // 32 slices' partials in flight, added in slice order
            float v[32];
#pragma unroll
            for (int u = 0; u < 32; ++u) v[u] = sb + u < S ? __ldcg(part + ((size_t)(sb + u) * M + m) * r + j) : 0.f;
#pragma unroll
            for (int u = 0; u < 32; ++u) t += v[u];
        }
        P.T[(size_t)m * P.t_ld + sg.t_off + j] = t;
    }
    if (threadIdx.x == 0) P.cnt[pj] = 0u;  // for the next call
}

// ---------------------------------------------------------------- stream ---
__global__ void __launch_bounds__(FTH, 2) fp4_stream_kernel(const __grid_constant__ Fp4Params P) {
    pdl_launch_dependents();
    __shared__ float4 red[FW][32][2];  // each warp's fragments: W0 x, U T
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
    const int b = blockIdx.x;
    int sp = 0;
    while (sp + 1 < P.nseg && b >= P.seg[sp + 1].blk_begin) ++sp;
    const Fp4Seg &S = P.seg[sp];
    const int row0 = (b - S.blk_begin) * 16;
    const int K = P.K, M = P.M, N = S.N;
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
    pdl_wait_primary();  // xh and T are the prep kernel's

    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    const bool xv = g < M;
    const __half *xr = P.xh + (size_t)(xv ? g : 0) * K + 32 * q;
    for (int kg0 = warp; kg0 < nkg; kg0 += FW * FKB) {
        if (kg0 != warp) load(kg0);
#pragma unroll
        for (int i = 0; i < FKB; ++i) {
            const int kg = kg0 + i * FW;
            if (kg >= nkg) break;
            uint4 xf[4];
#pragma unroll
            for (int t = 0; t < 4; ++t)
                xf[t] = xv ? __ldg(reinterpret_cast<const uint4 *>(xr + (size_t)kg * FKG) + t)
                           : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t xw[16] = {xf[0].x, xf[0].y, xf[0].z, xf[0].w, xf[1].x, xf[1].y, xf[1].z, xf[1].w,
                                     xf[2].x, xf[2].y, xf[2].z, xf[2].w, xf[3].x, xf[3].y, xf[3].z, xf[3].w};
            const uint32_t sc0 = e4m3x2_to_f16x2(sb0[i]), sc1 = e4m3x2_to_f16x2(sb1[i]);
            const uint32_t cw0[4] = {cb0[i].x, cb0[i].y, cb0[i].z, cb0[i].w};
            const uint32_t cw1[4] = {cb1[i].x, cb1[i].y, cb1[i].z, cb1[i].w};
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
                // elements 8 wi .. 8 wi + 7 of the lane's 32: block scale 0 for
                // the first 16, 1 for the last 16
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
                    mma_f16(acc[hh], a, xw[4 * wi + 2 * hh], xw[4 * wi + 2 * hh + 1]);
                }
            }
        }
    }

    // ---- U T over 32-column groups of the rank ----
    float acd[4] = {0.f, 0.f, 0.f, 0.f};
    const int r = S.r;
    for (int jg = warp; jg * 32 < r; jg += FW) {
        const int j = jg * 32 + 8 * q;  // this lane's eight rank columns
        const bool jv = j < r;
        const uint4 ulo = (jv && ok0) ? __ldg(reinterpret_cast<const uint4 *>(S.U + (size_t)(row0 + g) * r + j))
                                      : make_uint4(0u, 0u, 0u, 0u);
        const uint4 uhi = (jv && ok1) ? __ldg(reinterpret_cast<const uint4 *>(S.U + (size_t)(row0 + g + 8) * r + j))
                                      : make_uint4(0u, 0u, 0u, 0u);
        float t[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) t[e] = (jv && xv) ? __ldcg(P.T + (size_t)g * P.t_ld + S.t_off + j + e) : 0.f;
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
    red[warp][lane][0] = make_float4(acc[0][0] + acc[1][0], acc[0][1] + acc[1][1], acc[0][2] + acc[1][2],
                                     acc[0][3] + acc[1][3]);
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

// ------------------------------------------------------------------ host ---
size_t fp4_tpart_floats(const Fp4Params &p) { return (size_t)p.slices * p.M * (p.t_ld > 0 ? p.t_ld : 1); }

int fp4_prep_slices(int K) { return (K + kPrepRows - 1) / kPrepRows; }

cudaError_t launch_fp4(const Fp4Params &p, cudaStream_t stream) {
    int nr = 0;
    for (int i = 0; i < p.nseg; ++i) nr += p.seg[i].r > 0;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(FTH);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3((unsigned)(p.slices * (nr > 0 ? nr : 1)));
    cudaError_t e = cudaLaunchKernelEx(&cfg, fp4_prep_kernel, p);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((unsigned)p.total_blocks);
    return cudaLaunchKernelEx(&cfg, fp4_stream_kernel, p);
}

}  // namespace wl
