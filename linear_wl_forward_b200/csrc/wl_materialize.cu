// W_eff = diag(s) W0 + U V^T for one projection, in bf16 with fp32
// accumulation: the dense weight a theta bundle stands for ("Add a new model
// architecture", "Override the graph build", step 5: the precompute-outside
// form that rebuilds the weight once and then runs a plain matmul).  A weight
// is rebuilt once and reused, so this is a simple tiled kernel: a CTA computes
// a 64 x 64 tile of W_eff, staging 64-column slices of the tile's U rows and
// V rows in shared memory; each thread accumulates a 4 x 4 patch in fp32.
#include "wl_common.cuh"
#include "wl_internal.h"

namespace wl {
namespace {

constexpr int kTile = 64;
constexpr int kSlice = 64;  // rank columns staged per round

__global__ void __launch_bounds__(256) materialize_kernel(const __nv_bfloat16 *__restrict__ W0,
                                                          const float *__restrict__ s,
                                                          const __nv_bfloat16 *__restrict__ U,
                                                          const __nv_bfloat16 *__restrict__ V,
                                                          __nv_bfloat16 *__restrict__ Weff, int N, int K, int r) {
    pdl_launch_dependents();
    pdl_wait_primary();
    __shared__ float us[kSlice][kTile + 1];  // [j][row n]
    __shared__ float vs[kSlice][kTile + 1];  // [j][column k]
    const int n0 = blockIdx.y * kTile, k0 = blockIdx.x * kTile;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;  // 16 x 16 threads, 4 x 4 outputs each
    float acc[4][4] = {};
    for (int j0 = 0; j0 < r; j0 += kSlice) {
        for (int i = threadIdx.x; i < kTile * kSlice; i += 256) {
            const int row = i / kSlice, j = i - row * kSlice;
            const int n = n0 + row, k = k0 + row, jj = j0 + j;
            us[j][row] = (n < N && jj < r) ? __bfloat162float(U[(size_t)n * r + jj]) : 0.f;
            vs[j][row] = (k < K && jj < r) ? __bfloat162float(V[(size_t)k * r + jj]) : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int j = 0; j < kSlice; ++j) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = us[j][ty * 4 + i];
                b[i] = vs[j][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[i][c] = fmaf(a[i], b[c], acc[i][c]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int n = n0 + ty * 4 + i;
        if (n >= N) continue;
        const float sc = s[n];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int k = k0 + tx * 4 + c;
            if (k < K) {
                const size_t o = (size_t)n * K + k;
                Weff[o] = __float2bfloat16_rn(fmaf(sc, __bfloat162float(W0[o]), acc[i][c]));
            }
        }
    }
}

}  // namespace

cudaError_t launch_materialize(const __nv_bfloat16 *W0, const float *s, const __nv_bfloat16 *U,
                               const __nv_bfloat16 *V, __nv_bfloat16 *Weff, int N, int K, int r,
                               cudaStream_t stream) {
    dim3 grid((K + kTile - 1) / kTile, (N + kTile - 1) / kTile);
    if (grid.y > 65535u) return cudaErrorInvalidValue;  // N above 65535 * 64 rows
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, materialize_kernel, W0, s, U, V, Weff, N, K, r);
}

}  // namespace wl
