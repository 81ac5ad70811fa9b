// Host/device shared parameter blocks and the launchers behind the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/wl.h"

namespace wl {

constexpr int kMaxSeg = WL_MAX_PROJ;

// --------------------------------------------------------------- decode ----
// Streaming decode kernel: M <= WL_DECODE_MAX_M tokens.  The projections of a
// stacked call are concatenated into one row space [0, total_rows).
constexpr int kDecodeKC = 1024;       // K elements per row per stage (2 KB)
constexpr int kDecodeRowsPerStage = 8;  // one row per consumer warp
constexpr int kDecodeStages = 8;      // ring depth: 8 x 16 KB in flight per SM
constexpr int kDecodeRowsCap = 1024;  // rows per CTA (sizes the z partials)
constexpr int kDecodeThreads = 32 * (kDecodeRowsPerStage + 1);
constexpr int kTChunk = 128;          // V rows per block of the V^T x kernel

struct DecodeSeg {
    const __nv_bfloat16 *W0;
    const float *s;
    const __nv_bfloat16 *U;
    const __nv_bfloat16 *V;
    __nv_bfloat16 *y;
    int N;
    int r;
    int t_off;      // column offset of this projection's T slice
    int row_begin;  // first row in the concatenated row space
    int tblk_begin; // first block of the V^T x kernel for this projection
};

struct DecodeParams {
    DecodeSeg seg[kMaxSeg];
    int nseg;
    int M, K;
    int total_rows;
    int t_ld;       // row stride of T (sum of ranks)
    int r_max;
    int u_bulk;     // all U rows can be moved by 16-byte bulk copies
    int has_lowrank;
    const __nv_bfloat16 *x;
    float *T;       // M x t_ld fp32 (V^T x, written by the V^T x kernel)
    float *Tpart;   // per-block partial sums, [blocks][M][r_max]
    int *counters;  // one arrival counter per projection (self-resetting)
    int *status;
    unsigned long long timeout_ns;
};

size_t decode_smem_bytes(int M);
int decode_t_blocks(int K);
cudaError_t launch_decode(const DecodeParams &p, int num_sms, cudaStream_t stream);

// ----------------------------------------------------------------- GEMM ----
// tcgen05 GEMM: Y[m][n] = s[n] * sum_k A[m][k] B[n][k] + sum_j T[m][j] U[n][j].
constexpr int kGemmBM = 128;
constexpr int kGemmBK = 64;         // 128 bytes of bf16: one swizzle row
constexpr int kGemmMaxBN = 256;
constexpr int kGemmStages = 4;
constexpr int kGemmThreads = 192;   // producer, MMA, 4 epilogue warps

struct GemmSeg {
    const float *s;       // nullable: scale 1
    __nv_bfloat16 *y;
    int N;
    int ldy;
    int lr_blocks;        // low-rank K blocks (r_pad / 64), 0 = none
    int t_col;            // column of this segment's slice in T
    int tile_begin;
};

struct GemmParams {
    CUtensorMap tm_a;                // x (M x K) or, for T = x V, x
    CUtensorMap tm_t;                // T (M x t_cols) bf16
    CUtensorMap tm_b[kMaxSeg];       // W0_p (N_p x K)
    CUtensorMap tm_u[kMaxSeg];       // U_p (N_p x r)
    GemmSeg seg[kMaxSeg];
    int nseg;
    int M, K;
    int BN;
    int num_m_tiles;
    int num_tiles;
    int *status;
    unsigned long long timeout_ns;
};

size_t gemm_smem_bytes();
cudaError_t launch_gemm(const GemmParams &p, int num_sms, cudaStream_t stream);

// Vt[j][k] = V[k][j] for j < r, 0 for r <= j < r_pad (rows of the stacked
// transposed V, one projection per call).
cudaError_t launch_transpose_v(const __nv_bfloat16 *V, int K, int r, int r_pad,
                               __nv_bfloat16 *Vt, cudaStream_t stream);
// Copy U (N x r) into Upad (N x r_pad) with zero columns beyond r.
cudaError_t launch_pad_u(const __nv_bfloat16 *U, int N, int r, int r_pad,
                         __nv_bfloat16 *Upad, cudaStream_t stream);

// --------------------------------------------------------------- probes ----
cudaError_t launch_wait_probe(int *flag, int *status, unsigned long long limit_ns,
                              cudaStream_t stream);

}  // namespace wl
