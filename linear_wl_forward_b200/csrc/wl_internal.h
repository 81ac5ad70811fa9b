// Host/device shared parameter blocks and the launchers behind the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/wl.h"

namespace wl {

constexpr int kMaxSeg = WL_MAX_PROJ;

// ------------------------------------------------------------- prefetch ----
// Device ranges a call's kernels pull into L2 for the calls that follow it
// (wl_stacked_forward_prefetch): each range is trimmed on the host to its
// 16-byte-aligned interior, and the CTAs of the launch share the bytes out
// evenly, in order.
constexpr int kMaxPrefetch = WL_MAX_PREFETCH;
constexpr uint32_t kPrefetchPiece = 64 * 1024;  // bytes per bulk prefetch instruction

struct PrefetchList {
    const uint8_t *ptr[kMaxPrefetch];  // 16-byte aligned
    uint64_t bytes[kMaxPrefetch];      // multiples of 16
    uint64_t total;                    // sum of bytes
    int n;
};

// --------------------------------------------------------------- decode ----
// Streaming decode kernel: M <= WL_DECODE_MAX_M tokens.  The projections of a
// stacked call are concatenated into one list of 16-row blocks.
constexpr int kDecodeWarps = 8;
constexpr int kDecodeThreads = 32 * kDecodeWarps;
constexpr int kDecodeBlockRows = 16;      // rows of one MMA row block
constexpr int kDecodeChunkK = 64;         // K columns per TMA box (128 B, swizzled)
constexpr int kDecodeChunkBytes = kDecodeBlockRows * kDecodeChunkK * 2;  // 2 KB
constexpr int kDecodeMaxSlotChunks = 4;   // a ring slot holds up to 16 rows x 256 columns
constexpr int kDecodeMaxSlots = 4;        // ring slots per warp
constexpr int kDecodeTMaxFloats = 12288;  // M (rounded up to 8) * (sum of ranks) in shared memory
constexpr int kDecodeMaxLag = 3;          // grid T mode: blocks by which the U part of a block trails its W0 part
constexpr int kDecodeFusedMaxRank = 32;   // fused local T: largest rank (two 16-column tiles of T per warp)

// How a CTA obtains T = V^T x.
enum DecodeTMode : int {
    kTNone = 0,   // no projection has a delta
    kTLocal = 1,  // each CTA forms the T slices its rows need from all of V
    kTGrid = 2    // each CTA forms partial sums over a K slice; two grid-wide
                  // arrival counts later every CTA has the T slices it needs
};

struct DecodeSeg {
    const __nv_bfloat16 *W0;
    const float *s;
    const __nv_bfloat16 *U;
    const __nv_bfloat16 *V;
    __nv_bfloat16 *y;
    int N;
    int r;
    int t_off;      // column offset of this projection's T slice
    int blk_begin;  // first 16-row block of this projection in the call's block list
    int cta_begin;  // seg_split: first CTA of this projection
};

// Everything the decode kernel reads except the tensor maps.  The kernel
// copies it into shared memory once at the start: a parameter block is new
// for every launch, so reading it in place costs a chain of constant-cache
// misses right on the path after the wait for the previous kernel.
struct DecodeArgs {
    DecodeSeg seg[kMaxSeg];
    int nseg;
    int M, K;
    int total_blocks;
    int seg_split;    // CTAs are split over the projections in proportion to their blocks
    int t_ld;         // row stride of T (sum of ranks)
    int slot_chunks;  // 64-column chunks per ring slot (1 .. kDecodeMaxSlotChunks)
    int slots;        // ring slots per warp (1 .. kDecodeMaxSlots)
    int w3d;          // K % 64 == 0 and slot_chunks > 1: a full W0 slot is one 3-D box
    int u_bulk;       // every U is TMA-able (r % 8 == 0, 16-byte aligned)
    int t_mode;       // DecodeTMode
    int lag;          // kTGrid: the U part of block b runs in step b + lag
    int x_smem;       // x is staged in shared memory (rows padded to x_ld elements)
    int x_ld;
    int v_stage;      // each CTA bulk-copies the V rows it needs for T into shared memory
    int v_bytes;      // shared memory they need (largest over the CTAs)
    int v_in_ring;    // they sit in the ring's last slot level until T's sums are formed
    int u_stage;      // each CTA bulk-copies its blocks' U rows into shared memory (not through the ring)
    int u_bytes;      // shared memory they need (largest over the CTAs)
    int t_fused;      // kTLocal: T's MMAs run inside the first step's W0 part (sharing its x
                      // fragments) and every epilogue adds U T from the staged U rows
    const __nv_bfloat16 *x;
    float *Tpart;     // kTGrid: [grid][M][t_ld] partial sums, then [M][t_ld] final T
    unsigned int *sync;  // kTGrid: [0], [1] arrival counts, [2] departures; self-resetting
    int *status;
    unsigned long long timeout_ns;
};

struct DecodeParams {
    DecodeArgs a;
    PrefetchList pf;             // read by one thread per CTA, before the wait
    CUtensorMap tm_w[kMaxSeg];   // W0: 2-D {K, N}, box {64, 16}, 128-B swizzle
    CUtensorMap tm_w3[kMaxSeg];  // W0: 3-D {64, N, K/64}, box {64, 16, slot_chunks} (when w3d)
    CUtensorMap tm_u[kMaxSeg];   // U:  2-D {r, N}, box {64, 16} (when u_bulk)
};

// Host-side planning shared by every decode entry point.
struct DecodePlan {
    int grid;
    int small;           // the compact variant, two CTAs per SM (consecutive calls overlap)
    size_t smem;
    size_t tpart_bytes;  // scratch for kTGrid partial sums and final T (0 otherwise)
};
// Fills the block list, the CTA split, the tensor maps and the ring, T and
// shared-memory choices; returns WL_ERR_UNSUPPORTED if the shape cannot take
// the decode path (M above WL_DECODE_MAX_M, or M rounded up to 8 times the sum
// of ranks above kDecodeTMaxFloats).
// encode_maps = false plans without the tensor maps (host logic only: no
// driver call, the pointers are only checked for alignment).
wl_status plan_decode(DecodeParams &p, int num_sms, DecodePlan *plan, bool encode_maps = true);
cudaError_t launch_decode(const DecodeParams &p, const DecodePlan &plan, cudaStream_t stream);

// 2-D / 3-D bf16 tensor maps (128-byte swizzling unless swizzle128 is false);
// out-of-range reads give 0.
wl_status encode_map_2d(CUtensorMap *m, const void *ptr, uint64_t cols, uint64_t rows, uint64_t ld,
                        uint32_t box_cols, uint32_t box_rows, bool swizzle128 = true);
// Raw bytes viewed as 32-bit words: rows of `cols` words, `ld_bytes` apart
// (a multiple of 16), no swizzle.
wl_status encode_map_2d_u32(CUtensorMap *m, const void *ptr, uint64_t cols, uint64_t rows, uint64_t ld_bytes,
                            uint32_t box_cols, uint32_t box_rows);
// n fp32 values, boxes of `box`.
wl_status encode_map_1d_f32(CUtensorMap *m, const void *ptr, uint64_t n, uint32_t box);
wl_status encode_map_3d(CUtensorMap *m, const void *ptr, uint64_t d0, uint64_t d1, uint64_t d2,
                        uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1,
                        uint32_t b2, bool bytes_unswizzled = false);

// ----------------------------------------------------------- row stream ----
// Row-stream decode kernel for short calls (latency-bound: a few MB of
// weights).  Each CTA owns a group of up to kRowsMaxBlocks 16-row blocks of
// one projection and, with a cluster of c CTAs, 1/c of K; before the wait for
// the previous kernel its warps copy their share of W0 into shared memory
// (TMA tiles laid out as the lanes' MMA fragments) and V and U rows are
// bulk-copied there, and the partial sums of the c CTAs meet over
// distributed shared memory.
constexpr int kRowsWarps = 8;
constexpr int kRowsThreads = 32 * kRowsWarps;
constexpr int kRowsKGroup = 32;     // K columns per warp step (two m16n8k16 MMAs)
constexpr int kRowsMaxBlocks = 4;   // 16-row blocks per CTA
constexpr int kRowsMaxRank = 64;    // four 16-column tiles of T
constexpr int kRowsMaxCluster = 4;  // CTAs sharing one row group along K
constexpr int kRowsXPad = 32;       // elements of padding per staged x row (bank spread)

struct RowsSeg {
    const __nv_bfloat16 *W0;
    const float *s;
    const __nv_bfloat16 *U;
    const __nv_bfloat16 *V;
    __nv_bfloat16 *y;
    int N, r;
    int grp_begin;  // first row group (cluster) of this projection
    int nb;         // 16-row blocks per row group (the last group may have fewer)
};

struct RowsParams {
    CUtensorMap tm_w[kMaxSeg];  // W0_p: 2-D {K, N_p}, box {32, 16 nb_p}, no swizzle
    RowsSeg seg[kMaxSeg];
    int nseg;
    int M, K;
    int c;       // CTAs per cluster: the K slices of one row group
    int ks;      // K columns per slice (a multiple of kRowsKGroup)
    int ngroups; // row groups (clusters) in the grid
    int nb_max;  // largest nb over the projections
    int r_max;
    // shared memory offsets (bytes) and total
    uint32_t off_w, off_v, off_u, off_x, off_zc, off_tc, off_tf, off_s, off_bar, smem;
    const __nv_bfloat16 *x;
    int *status;
    unsigned long long timeout_ns;
    PrefetchList pf;
};

// Plans a call for the row-stream kernel on a GPU with num_sms SMs; returns
// WL_ERR_UNSUPPORTED when it does not fit (M > 16, a rank above
// kRowsMaxRank or not a multiple of 8, U / V not 16-byte aligned, more than
// kRowsMaxBlocks blocks per CTA, or the shared-memory budget).  encode_maps =
// false plans without the tensor maps (host logic only).
wl_status plan_rows(RowsParams &p, int M, int K, const wl_proj *projs, int P, int num_sms,
                    bool encode_maps = true);
cudaError_t launch_rows(const RowsParams &p, cudaStream_t stream);

// -------------------------------------------------------- NVFP4 decode ----
// Decode with W0 stored as NVFP4 (E2M1 codes, E4M3 scales per 16 elements,
// fp32 tensor scale).  A prep launch forms T = V^T x and a permuted f16 copy
// of x; then one of two weight-stream launches:
//  * ring (K % 256 == 0, every rank <= 256): persistent, one CTA per SM; a
//    producer warp streams (block, stage) units through a shared-memory ring
//    by TMA, the units split evenly over the CTAs;
//  * blocks (otherwise): one CTA per 16-row block, loads straight into
//    registers.
constexpr int kFp4KGroup = 128;  // K columns per warp step; K must be a multiple
constexpr int kFp4MaxM = 8;      // tokens
constexpr int kFp4StageKG = 16;  // k-groups per ring stage (2048 columns)
constexpr int kFp4RingMaxRank = 256;
constexpr int kFp4RingMaxStages = 16;

struct Fp4Seg {
    const uint8_t *codes;   // N x K/2
    const uint8_t *scales;  // N x K/16
    float ts;               // tensor scale
    const float *s;
    const __nv_bfloat16 *U;
    const __nv_bfloat16 *V;
    __nv_bfloat16 *y;
    int N, r;
    int blk_begin;  // first 16-row block of this projection
    int t_off;      // column of this projection's slice in T
    long long ub;   // ring: first unit of this projection
    int upb;        // ring: units per block (stages, plus one for U when r > 0)
};

struct Fp4Params {
    Fp4Seg seg[kMaxSeg];
    CUtensorMap tm_c[kMaxSeg];  // ring: codes as 32-bit words, box 16 rows x 512 bytes
    CUtensorMap tm_s[kMaxSeg];  // ring: scales as 32-bit words, box 16 rows x 64 bytes
    CUtensorMap tm_u[kMaxSeg];  // ring: U as 32-bit words, box 16 rows x 2r bytes
    CUtensorMap tm_sv[kMaxSeg]; // ring: s, boxes of 16 values
    int nseg;
    int M, K;
    int Mp;       // token rows of the permuted x (M, rounded up to even above 1)
    int total_blocks;
    int t_ld;     // sum of ranks
    int nr;       // projections with a delta
    // prep: T over slices of K, summed in groups of kFp4GroupSlices then over groups
    int slices, kr, ngrp;
    const __nv_bfloat16 *x;
    __half *xq;           // permuted f16 x (written by the prep launch)
    float *Tpart;         // [slices][M][t_ld]
    float *Gpart;         // [ngrp][M][t_ld]
    float *T;             // [M][t_ld]
    unsigned int *cnt;    // [nr][ngrp] group counters, then [nr] projection counters (zeroed, self-resetting)
    // ring
    int bf16;             // 1: W0 in bf16 (codes = the bf16 rows, no scales, tensor scale 1); ring stream only
    int ring;             // 1: ring stream, 0: block stream
    int grid, ns, slot_bytes, smem, nst;
    int ku;               // k-units per stage (128-column groups for NVFP4, 32-column for bf16)
    long long utot;
    float2 *parts;        // [grid][2][16 * kFp4MaxM] partial (z, d) of blocks split between CTAs
    unsigned int *bcnt;   // [total_blocks] CTAs done with a split block (zeroed, self-resetting)
    int *status;
    unsigned long long timeout_ns;
};

constexpr int kFp4GroupSlices = 16;
constexpr int kFp4PrepMaxRows = 256;

// Fills slices/kr/ngrp/Mp and, for the ring stream (encode_maps), the tensor
// maps and ring geometry; p.seg/nseg/M/K/t_ld/nr must be set.
wl_status plan_fp4(Fp4Params &p, int num_sms, bool encode_maps = true);
size_t fp4_xq_halves(const Fp4Params &p);
cudaError_t launch_fp4(const Fp4Params &p, cudaStream_t stream);

// ----------------------------------------------------------------- GEMM ----
// tcgen05 GEMM: Y[m][n] = s[n] * sum_k A[m][k] B[n][k] + sum_j T[m][j] U[n][j].
constexpr int kGemmBM = 128;
constexpr int kGemmBK = 64;         // 128 bytes of bf16: one swizzle row
constexpr int kGemmMaxBN = 256;
constexpr int kGemmMaxStages = 12;
constexpr int kGemmSwapMaxM = 16;   // swap-AB mode up to this many tokens (measured: at 64 the 128-row x tiles win)
constexpr int kGemmMaxKSplit = 8;   // K ranges per output tile in swap mode
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
    int swap;         // few-token mode: A = 128-row W0 (or U) tiles, B = x (or T) tiles of mp rows
    int mp;           // swap: B rows, the token count rounded up to 16 (the MMA's N)
    int ksplit;       // K-block ranges per output tile (1 unless swap); their sums meet in `part`
    int kb_split;     // K blocks per range
    float *part;      // swap, ksplit > 1: [ksplit][tiles][mp][128] partial W0 x sums, then [tiles][mp][128] U T
    unsigned int *tile_cnt;  // swap, ksplit > 1: per-tile arrival counts, self-resetting (zeroed at allocation)
    int stages;       // pipeline depth (set_gemm_stages)
    int stage_bytes;
    int num_m_tiles;
    int num_tiles;
    int *status;
    unsigned long long timeout_ns;
    PrefetchList pf;
};

void set_gemm_stages(GemmParams &p);
size_t gemm_smem_bytes(const GemmParams &p);
cudaError_t launch_gemm(const GemmParams &p, int num_sms, cudaStream_t stream);

// Vt[row_p + j][k] = V_p[k][j] for j < r_p, 0 for r_p <= j < r_pad_p: the
// stacked transposed V of every projection of a call, in one launch.
struct TransposeVArgs {
    const __nv_bfloat16 *V[kMaxSeg];
    int r[kMaxSeg];
    int r_pad[kMaxSeg];
    int row[kMaxSeg];  // first row of projection p in Vt
    int n;
    int K;
    __nv_bfloat16 *Vt;
};
cudaError_t launch_transpose_v(const TransposeVArgs &a, cudaStream_t stream);
// Copy U (N x r) into Upad (N x r_pad) with zero columns beyond r.
cudaError_t launch_pad_u(const __nv_bfloat16 *U, int N, int r, int r_pad,
                         __nv_bfloat16 *Upad, cudaStream_t stream);

// ---------------------------------------------------------- materialize ----
// Weff = diag(s) W0 + U V^T (bf16 out, fp32 accumulation), all N x K row-major.
cudaError_t launch_materialize(const __nv_bfloat16 *W0, const float *s, const __nv_bfloat16 *U,
                               const __nv_bfloat16 *V, __nv_bfloat16 *Weff, int N, int K, int r,
                               cudaStream_t stream);

// ----------------------------------------------------------- wait limit ----
// Time limit of every device-side wait the forward kernels make (2 s unless
// wl_set_wait_limit changed it).
unsigned long long wait_limit_ns();

// --------------------------------------------------------------- probes ----
cudaError_t launch_wait_probe(int *flag, int *status, unsigned long long limit_ns,
                              cudaStream_t stream);

}  // namespace wl
