/*
 * wl.h -- C ABI of the B200 theta-bundle linear ("weightless" linear).
 *
 * A theta bundle replaces one dense projection weight by a shared block W0, a
 * per-output-row scale s and a rank-r delta (U, V), and the layer computes
 *
 *     y = s (.) (W0 x) + U (V^T x)
 *
 * ("Add a new model architecture", introduction: the theta bundle rebuilds one
 * projection's weight as y = s.(W0 x) + U.(V^T x)).  W0 is shared by all layers
 * of a band ("Quality": G = shared_blocks sets how many layers share one W0);
 * s, U, V belong to one layer.
 *
 * Conventions for every entry point below
 * ---------------------------------------
 *  - Element types: wl_bf16 is a raw IEEE bfloat16 bit pattern; s is float32.
 *  - Layouts are row-major: x is M x K (one token per row), W0 is N x K (the
 *    Linear.weight orientation: rows are outputs), U is N x r, V is K x r,
 *    y is M x N.  In row-major terms the layer computes Y = X W0^T scaled per
 *    column n by s[n], plus (X V) U^T.
 *  - Pointers passed to the forward calls are DEVICE pointers on the current
 *    CUDA device, owned by the caller; the library never frees or retains them
 *    beyond the call's kernels.
 *  - Forward calls are asynchronous on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream).  They do not synchronise the host.  They need
 *    scratch on the device (the low-rank product V^T x and, for large M, a
 *    transposed copy of V); it comes from a library-owned per-device pool that
 *    grows on first use of a larger size and is then reused, so calls of a
 *    repeated shape do not allocate.  Calls that overlap on the GPU (different
 *    streams, or different host threads) share that pool and must not run
 *    concurrently; calls on one stream are always safe.
 *  - Accumulation is fp32 (tensor cores or CUDA cores); y is rounded once to
 *    bf16 (round to nearest even).  No atomics take part in any sum, so results
 *    are reproducible run to run.
 *  - Errors are returned, never aborted on: argument problems are detected on
 *    the host before anything is launched; launch failures give WL_ERR_CUDA; a
 *    device-side wait that exceeded its time limit (2 s, see
 *    wl_set_wait_limit) is reported later by wl_last_device_status().  A call
 *    whose wait gave up leaves its outputs partly unwritten and may leave a
 *    grid-wide arrival count set, so the results of the calls issued after it
 *    are undefined until wl_last_device_status() has returned the error (it
 *    clears the counts).
 *  - Some kernels wait for one another's CTAs inside one launch (the decode
 *    kernel's grid-wide V^T x exchange; the GEMM's K-range sums are collected
 *    by the last CTA to arrive, without waiting).  Those launches never have
 *    more CTAs than the SMs can hold at once, so on a GPU shared with other
 *    processes a CTA that cannot become resident within the wait limit makes
 *    the call fail with WL_ERR_TIMEOUT instead of hanging.
 */
#ifndef WL_H_
#define WL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t wl_bf16;

typedef enum {
    WL_OK = 0,
    WL_ERR_INVALID_ARG = 1, /* null pointer where data is needed, negative size   */
    WL_ERR_ALIGNMENT = 2,   /* K % 8 != 0, or x / W0 not 16-byte aligned          */
    WL_ERR_UNSUPPORTED = 3, /* r > WL_MAX_RANK, P > WL_MAX_PROJ, no sm_100 device */
    WL_ERR_CUDA = 4,        /* a CUDA runtime call or a kernel launch failed      */
    WL_ERR_TIMEOUT = 5,     /* a device-side wait gave up (see wl_last_device_status) */
    WL_ERR_NOMEM = 6,       /* scratch pool could not grow                          */
    WL_ERR_NOT_CONVERGED = 7 /* host SVD hit its sweep limit (outputs are filled)   */
} wl_status;

#define WL_MAX_RANK 1024
#define WL_MAX_PROJ 8

/* One projection of a stacked call ("Quality (Gemma 4 31B)", "Kernel
 * optimizations", GEMM path item 1: q/k/v -- or gate/up -- share x).
 * All pointers are device pointers.  U and V may be NULL iff r == 0. */
typedef struct {
    const wl_bf16 *W0; /* N x K, row-major, 16-byte aligned            */
    const float *s;    /* N                                            */
    const wl_bf16 *U;  /* N x r, row-major                             */
    const wl_bf16 *V;  /* K x r, row-major                             */
    wl_bf16 *y;        /* M x N, row-major (output)                    */
    int N;             /* output rows of this projection, >= 0         */
    int r;             /* rank of the delta, 0 <= r <= WL_MAX_RANK     */
} wl_proj;

/* Which kernels a forward call uses.  WL_PATH_AUTO takes the persistent ring
 * for calls of at most 8 tokens whose weights total at least 64 MB when the
 * call fits it; else a
 * decode kernel for M <= 4, and for M <= WL_DECODE_MAX_M when the call's
 * projections total fewer than 8192 output rows; otherwise the tensor-core
 * GEMM.  Of the two decode
 * kernels it takes the row-stream one whenever the call fits it (short calls:
 * at most four 16-row blocks of W0 per SM, every rank <= 64 and a multiple of
 * 8, U and V 16-byte aligned), else the weight-streaming one.  The others
 * exist so tests and benchmarks can exercise each kernel on any shape. */
typedef enum {
    WL_PATH_AUTO = 0,
    WL_PATH_DECODE = 1, /* weight-streaming kernel (bulk copies + warp MMA), 1 <= M <= WL_DECODE_MAX_M */
    WL_PATH_GEMM = 2,   /* tcgen05 tensor-core GEMM with the fused low-rank epilogue */
    WL_PATH_ROWS = 3,   /* row-stream decode kernel (register-fed warp MMA, K split over CTA
                           clusters) for short calls; WL_ERR_UNSUPPORTED for calls it does not fit */
    WL_PATH_RING = 4    /* persistent ring decode (a V^T x launch, then one CTA per SM streaming
                           16-row x 1536-column (M <= 2) or x 1024-column weight tiles by TMA,
                           the call's work split evenly over the SMs) for 1 <= M <= 8, ranks
                           <= 256 and multiples of 8, U, V and s 16-byte aligned;
                           WL_ERR_UNSUPPORTED otherwise */
} wl_path;

#define WL_DECODE_MAX_M 16

/* y = s (.) (W0 x) + U (V^T x) for one projection of one layer
 * ("Add a new model architecture", introduction; the delta is never
 * materialised as U V^T).
 *   x  : device, M x K bf16 row-major, 16-byte aligned
 *   W0 : device, N x K bf16 row-major, 16-byte aligned
 *   s  : device, N fp32
 *   U  : device, N x r bf16 row-major (NULL iff r == 0)
 *   V  : device, K x r bf16 row-major (NULL iff r == 0)
 *   y  : device, M x N bf16 row-major (written)
 * M, N >= 0 (0 is a no-op), K >= 0 with K % 8 == 0 (K == 0 writes y = 0),
 * 0 <= r <= WL_MAX_RANK.  Asynchronous on `stream` (cudaStream_t).
 * Ordering: the decode kernel is launched with programmatic dependent launch
 * and starts streaming W0, U, V and s while the previous kernel in the stream
 * still runs (x, y and the scratch are touched only after that kernel has
 * finished).  So W0, s, U and V must not be the outputs of the immediately
 * preceding forward call of this library on the same stream; outputs of any
 * other kernel are safe. */
wl_status wl_linear_forward(const wl_bf16 *x, const wl_bf16 *W0, const float *s,
                            const wl_bf16 *U, const wl_bf16 *V, wl_bf16 *y,
                            int M, int N, int K, int r, void *stream);

/* Several projections against one shared x in one pass ("Quality (Gemma 4
 * 31B)", "Kernel optimizations", GEMM path item 1: one fused W0 + V product and
 * a block-diagonal U product instead of one call per child).  projs is a HOST
 * array of P (1 <= P <= WL_MAX_PROJ) descriptors whose pointers are device
 * pointers; every projection has the same K.  Projection p writes its own
 * y_p (M x N_p), using only its own s_p, U_p and V_p.  Same conventions and
 * errors as wl_linear_forward. */
wl_status wl_stacked_forward(const wl_bf16 *x, int M, int K, const wl_proj *projs,
                             int P, void *stream);

/* wl_stacked_forward with an explicit kernel choice (see wl_path).
 * WL_PATH_DECODE and WL_PATH_ROWS require M <= WL_DECODE_MAX_M (else
 * WL_ERR_UNSUPPORTED); WL_PATH_ROWS also the limits of that kernel. */
wl_status wl_forward_ex(const wl_bf16 *x, int M, int K, const wl_proj *projs, int P,
                        wl_path path, void *stream);

/* A device range for wl_stacked_forward_prefetch. */
typedef struct {
    const void *ptr; /* device address (any alignment)                   */
    size_t bytes;    /* length; 0 is allowed and ignored                 */
} wl_range;

#define WL_MAX_PREFETCH 32

/* wl_forward_ex that also pulls `prefetch` (a HOST array of n ranges of
 * device memory, 0 <= n <= WL_MAX_PREFETCH; NULL iff n == 0) into L2 while
 * the call runs.  A decode step runs a fixed sequence of projections whose
 * weights do not change, so each call can name the weights of the call (or
 * calls) that follow it: those then start from L2 instead of HBM, and the
 * HBM stream of one call overlaps the arithmetic and epilogue of the one
 * before.  The pages name the cost this hides ("Quality (Gemma 4 31B)",
 * "Kernel optimizations": kernel launch overhead at batch-size-1 decode, and
 * the custom op being memory-bound at small dimensions).
 * Each range is trimmed to its 16-byte-aligned interior (so no byte outside
 * it is touched); the call's kernels share the bytes out over their CTAs and
 * issue them at their start, before waiting for the previous kernel in the
 * stream.  A prefetch moves data into L2 only, and L2 is coherent for the
 * whole device, so it never changes any result: ranges may hold anything,
 * including buffers other kernels are writing.  Keep the total well below
 * the 126 MB L2 (a few calls' weights).  Errors: those of wl_forward_ex;
 * WL_ERR_INVALID_ARG for n < 0, n > WL_MAX_PREFETCH, a NULL array with
 * n > 0, or a NULL range pointer with bytes > 0. */
wl_status wl_stacked_forward_prefetch(const wl_bf16 *x, int M, int K, const wl_proj *projs, int P,
                                      wl_path path, const wl_range *prefetch, int n,
                                      void *stream);

/* wl_linear_forward for callers that cannot allocate device memory while they
 * run: code living inside a pre-planned memory arena (an inference engine
 * whose allocator owns the device), callers under a hard memory budget, or
 * host threads that must not take the driver's allocation locks on a hot path.
 * The pages have no counterpart; it exists for these deployments only.
 *
 * Same arguments, layouts and conventions as wl_linear_forward, restricted to
 * the decode path: 1 <= M <= WL_DECODE_MAX_M (M == 0 or N == 0 is a no-op).
 * Scratch comes from one 4 MiB array in the library's device image that every
 * GPU loading the library keeps until the process exits; this entry point
 * never calls cudaMalloc, cudaFree or any allocating routine.  The scratch a
 * call needs is 256 B of counters plus, when V is large enough that the CTAs
 * share the work of V^T x, (grid+1)*M*r*4 B of partial sums (grid <= the SM
 * count: 149*M*r*4 B on a 148-SM B200).  A call needing more than 4 MiB
 * returns WL_ERR_UNSUPPORTED, as do M > WL_DECODE_MAX_M and shapes the decode
 * kernel cannot take (M rounded up to 8, times r, above 12288).
 *  - The first call on each device resolves the array's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before any stream capture.
 *  - All calls share the one array, which keeps the previous call's contents;
 *    each call clears the parts that must start at zero on its own stream.
 *    Calls that overlap on the GPU (different streams or host threads) race on
 *    the array: serialise them.
 *  - A device-side wait that times out here is recorded in the array's own
 *    status word, which wl_noalloc_last_status() reads (not
 *    wl_last_device_status()); each call clears the array's arrival counts
 *    before its kernel runs, and the status word keeps the first error until
 *    it is read. */
wl_status wl_linear_forward_noalloc(const wl_bf16 *x, const wl_bf16 *W0, const float *s,
                                    const wl_bf16 *U, const wl_bf16 *V, wl_bf16 *y,
                                    int M, int N, int K, int r, void *stream);

/* Synchronises `stream`, then returns the status word of
 * wl_linear_forward_noalloc's array on the current device: WL_OK, or the
 * first error one of its calls recorded (WL_ERR_TIMEOUT from a device-side
 * wait that gave up) since the word was last read with an error.  After an
 * error it clears the array's status word and arrival counts.  Makes no
 * allocation; like the forward, its first call on a device looks up the
 * array's address. */
wl_status wl_noalloc_last_status(void *stream);

/* One projection of an NVFP4 call: W0 stored as 4-bit codes with block
 * scales, the encoding wl_quantize_nvfp4 produces ("Compression", "NVFP4:
 * 3.18x smaller weights": packed 4-bit weights, one float8_e4m3fn scale per 16
 * elements, 0.5625 bytes per element).  Device pointers. */
typedef struct {
    const uint8_t *codes;  /* N x K/2 bytes, row-major: FP4 E2M1, element 2i in the
                              low nibble of byte i; 16-byte aligned             */
    const uint8_t *scales; /* N x K/16 bytes, row-major: FP8 E4M3 scale of each
                              16-element block along K; 2-byte aligned          */
    float tensor_scale;    /* > 0: dequantised element = e2m1 * e4m3 * this     */
    const float *s;        /* N                                              */
    const wl_bf16 *U;      /* N x r row-major, 16-byte aligned (NULL iff r == 0) */
    const wl_bf16 *V;      /* K x r row-major, 16-byte aligned (NULL iff r == 0) */
    wl_bf16 *y;            /* M x N row-major (output)                         */
    int N;                 /* output rows, >= 0                                */
    int r;                 /* rank, 0 <= r <= WL_MAX_RANK, r % 8 == 0          */
} wl_proj_nvfp4;

#define WL_NVFP4_MAX_M 8

/* The stacked forward with NVFP4 shared blocks: for each projection
 *   y_p = s_p (.) (W0_p x) + U_p (V_p^T x),  W0_p the dequantised weight,
 * computed as decode (1 <= M <= WL_NVFP4_MAX_M): the tensor scale multiplies
 * s, the codes and block scales are expanded to f16 (an E2M1 value times an
 * E4M3 scale is exact in f16) and multiplied with x rounded to f16 on the
 * tensor cores, fp32 accumulation; U V^T x as in the bf16 path; y rounded once
 * to bf16.  x is read as bf16 and rounded to f16 (round to nearest even),
 * which is exact for |x| in [2^-14, 65504] -- the activations' range here.
 * Two kernel launches (V^T x with x in f16, then the weight stream: a
 * persistent TMA ring over all SMs when K % 256 == 0, every rank is at most
 * 256 and every scales pointer is 16-byte aligned, else one CTA per 16 rows);
 * scratch from the same pool as the other forward calls.  Results are
 * reproducible for a given call shape and GPU.  Errors: those of
 * wl_stacked_forward; WL_ERR_ALIGNMENT unless K % 128 == 0, codes are 16-byte
 * and scales 2-byte aligned, and every rank is a multiple of 8 with U and V
 * 16-byte aligned; WL_ERR_INVALID_ARG for a tensor scale that is not > 0 and
 * finite; WL_ERR_UNSUPPORTED for M > WL_NVFP4_MAX_M.  Device-side waits are
 * bounded as in the other calls (wl_last_device_status). */
wl_status wl_stacked_forward_nvfp4(const wl_bf16 *x, int M, int K, const wl_proj_nvfp4 *projs, int P,
                                   void *stream);

/* What wl_stacked_forward_nvfp4 would launch for a call: the host-side plan,
 * made without a GPU (no tensor maps, no launch).  The pointers in `projs` are
 * only checked (null, alignment), never dereferenced; `num_sms` stands for the
 * device's SM count.  Errors as wl_stacked_forward_nvfp4's argument checks;
 * all-zero for a call with nothing to launch. */
typedef struct {
    int ring;          /* 1: persistent TMA ring stream, 0: one CTA per 16 rows */
    int grid;          /* CTAs of the weight stream                            */
    int stages;        /* ring slots per CTA (ring only)                       */
    int slot_bytes;    /* bytes of one ring slot (ring only)                   */
    int smem_bytes;    /* dynamic shared memory per CTA (ring only)            */
    long long units;   /* (block, stage) units split over the CTAs (ring only) */
    int prep_slices;   /* slices of K in the V^T x launch                      */
    int prep_rows;     /* rows of V per slice                                  */
    int prep_grid;     /* CTAs of the V^T x launch                             */
} wl_nvfp4_plan;

wl_status wl_describe_nvfp4_plan(int M, int K, const wl_proj_nvfp4 *projs, int P, int num_sms,
                                 wl_nvfp4_plan *out);

/* Host-side decomposition of L dense layer weights into theta bundles
 * ("Quality", "Why sharing fails": band-mean W0, per-row scale s, low-rank
 * residual; "Add a new model architecture", "Decompose HF weights" step 4).
 *   W             : host, L x N x K fp32 (layer-major, each N x K row-major)
 *   band_of_layer : host, L ints in [0, G), or NULL for contiguous equal bands
 *                   band(l) = floor(l * G / L)
 *   W0 (out)      : host, G x N x K fp32 -- mean of each band's layers (zero
 *                   for a band with no layers)
 *   s  (out)      : host, L x N fp32 -- least-squares per-row scale
 *                   <W_l[n], W0[n]> / ||W0[n]||^2 (1 where W0[n] = 0)
 *   U  (out)      : host, L x N x r fp32 -- left singular vectors times
 *                   singular values of R_l = W_l - diag(s_l) W0
 *   V  (out)      : host, L x K x r fp32 -- right singular vectors of R_l
 *                   (columns beyond rank(R_l) are zero)
 *   rel_err (out) : host, L doubles, may be NULL -- relative Frobenius error
 *                   of diag(s) W0 + U V^T against W_l, in fp64 from the fp32
 *                   factors
 * Computes in fp64 on the calling thread, synchronously; the SVD is a
 * one-sided Jacobi iteration, stopped when every column pair is orthogonal to
 * the rounding level of its dot products (m times the fp64 unit roundoff, m
 * the column length) or after 80 sweeps.  Returns WL_ERR_INVALID_ARG for null
 * pointers, L, N, K, G < 1, r < 0 or a band index outside [0, G);
 * WL_ERR_NOMEM if host memory runs out; WL_ERR_NOT_CONVERGED (every output
 * still written, from the last sweep) if some layer's iteration reached the
 * sweep limit. */
wl_status wl_decompose(const float *W, int L, int N, int K, int G, int r,
                       const int *band_of_layer, float *W0, float *s, float *U,
                       float *V, double *rel_err);

/* wl_decompose followed by `iters` rounds of alternating least squares over
 * the band-mean start ("Quality (Gemma 4 31B)", "ALS optimization barely
 * helps": ALS tried as an improvement over the mean W0; the pages name the
 * method, not its steps).  One round makes three exact least-squares updates
 * of the total squared residual sum_l ||W_l - diag(s_l) W0 - U_l V_l^T||_F^2,
 * each over its own unknowns with the others fixed:
 *   1. W0_b[n] = sum_{l in b} s_l[n] (W_l[n] - (U_l V_l^T)[n]) / sum_{l in b} s_l[n]^2
 *      (the row is kept when every s_l[n] of the band is 0);
 *   2. s_l[n] = <W_l[n] - (U_l V_l^T)[n], W0_b[n]> / ||W0_b[n]||^2 (1 for a zero row);
 *   3. U_l V_l^T = rank-r truncated SVD of W_l - diag(s_l) W0_b.
 * So the total residual never grows.  iters = 0 is wl_decompose.  Same
 * arguments, layouts, outputs and errors as wl_decompose (iters < 0 is
 * WL_ERR_INVALID_ARG); the factors are carried in fp64 between rounds. */
wl_status wl_decompose_als(const float *W, int L, int N, int K, int G, int r,
                           const int *band_of_layer, int iters, float *W0, float *s,
                           float *U, float *V, double *rel_err);

/* ||W - (diag(s) W0 + U V^T)||_F / ||W||_F for one layer, host pointers, fp64
 * ("Quality": relative Frobenius error of diag(s).W0 + U.V^T against the true
 * weight).  Returns a negative value for invalid arguments. */
double wl_relative_frobenius_error(const float *W, const float *W0, const float *s,
                                   const float *U, const float *V, int N, int K, int r);

/* W_eff = diag(s) W0 + U V^T: the dense weight a theta bundle stands for,
 * rebuilt once so later calls can run the plain dense product ("Add a new
 * model architecture", "Override the graph build", step 5: the
 * precompute-outside path).  A dense forward is then wl_linear_forward with
 * W0 = W_eff, s = 1 and r = 0.
 *   W0 : device, N x K bf16 row-major       s : device, N fp32
 *   U  : device, N x r bf16 row-major       V : device, K x r bf16 row-major
 *   W_eff : device, N x K bf16 row-major (written; must not overlap the inputs)
 * fp32 accumulation, one rounding to bf16.  N, K, r >= 0 (N or K == 0 is a
 * no-op), r <= WL_MAX_RANK; U and V may be NULL iff r == 0.  Asynchronous on
 * `stream`.  Returns WL_ERR_INVALID_ARG for null pointers or negative sizes. */
wl_status wl_materialize_weight(const wl_bf16 *W0, const float *s, const wl_bf16 *U,
                                const wl_bf16 *V, wl_bf16 *W_eff, int N, int K, int r,
                                void *stream);

/* NVFP4 encoding of a weight for 4-bit weight streaming ("Compression",
 * section "NVFP4: 3.18x smaller weights": packed 4-bit weights plus one
 * float8_e4m3fn block scale per 16 elements, 0.5625 bytes per element,
 * quantised at load time).  Host memory, synchronous:
 *   W      : N x K fp32, row-major, finite
 *   codes  : N x K/2 bytes (written): FP4 E2M1 codes, element 2i in the low
 *            nibble of byte i, 2i + 1 in the high nibble
 *   scales : N x K/16 bytes (written): FP8 E4M3 scale of each 16-element
 *            block along K
 *   tensor_scale : > 0 to use as given; 0 to take max|W| / (6 * 448) rounded
 *            to fp32 (1 for an all-zero W); the value used is written to
 *            *tensor_scale_out
 * Dequantised element: e2m1(code) * e4m3(scale) * tensor scale.  Block
 * scale = max|w| of the block / (6 * tensor scale) and code = w / (block
 * scale * tensor scale), both in fp64, rounded to nearest-even and saturated
 * (448, 6); a block whose scale rounds to zero gets zero codes.
 * Returns WL_ERR_ALIGNMENT unless K % 16 == 0, WL_ERR_INVALID_ARG for
 * negative sizes, null buffers, a negative or infinite tensor_scale or a
 * non-finite W, WL_ERR_UNSUPPORTED if the host's floating-point rounding
 * mode is not round-to-nearest. */
wl_status wl_quantize_nvfp4(const float *W, int N, int K, float tensor_scale, uint8_t *codes,
                            uint8_t *scales, float *tensor_scale_out);

/* What the decode kernel would do with a call: the host-side plan, made
 * without a GPU (no tensor maps, no launch).  The pointers in `projs` are
 * checked for NULL and alignment only, never dereferenced, so stand-in
 * values describe a call before its buffers exist.  t_mode: 0 = no delta,
 * 1 = local (each CTA forms its T slices from the staged V rows), 2 = grid
 * (partial sums over K slices meet through two grid-wide counts). */
typedef struct {
    int auto_decode;  /* WL_PATH_AUTO takes the decode kernel for this call  */
    int grid;         /* CTAs, at most one per SM (two for compact calls)    */
    int compact;      /* the two-CTA/SM variant (<= 110 KB shared memory)     */
    long long smem_bytes; /* dynamic shared memory per CTA                  */
    int t_mode;       /* see above                                          */
    int t_fused;      /* T formed inside the first step's W0 MMAs           */
    int seg_split;    /* CTAs shared out among the stacked projections      */
    int slots;        /* ring slots per warp                                */
    int slot_chunks;  /* 64-column W0 chunks per slot                       */
    int x_smem;       /* x staged in shared memory                          */
    int v_stage;      /* the V rows for T staged in shared memory           */
    int v_in_ring;    /* ... in the ring's last slot level                  */
    int u_stage;      /* the U rows of the CTA's blocks staged              */
    int lag;          /* grid mode: steps by which a block's U part trails  */
} wl_decode_plan;

/* Fills *out for the call (M tokens, K, P projections as wl_stacked_forward
 * takes them) on a GPU with num_sms SMs.  out->auto_decode is set whenever
 * the arguments are valid.  Returns WL_ERR_UNSUPPORTED for shapes the decode
 * kernel declines (M outside 1..WL_DECODE_MAX_M, K < 8, too many T values),
 * and the argument errors of wl_stacked_forward. */
wl_status wl_describe_decode_plan(int M, int K, const wl_proj *projs, int P, int num_sms,
                                  wl_decode_plan *out);

/* The row-stream kernel's host-side plan for a call (see WL_PATH_ROWS), made
 * without a GPU; the pointers in `projs` are checked for NULL and alignment
 * only.  Output rows are cut into 16-row blocks, the blocks of each
 * projection into row groups of at most nb_max blocks, and each row group is
 * owned by a cluster of `cluster` CTAs that split K into slices of
 * k_slice columns. */
typedef struct {
    int grid;         /* CTAs (row groups x cluster), at most num_sms        */
    int cluster;      /* CTAs per cluster (1, 2 or 4)                        */
    int row_groups;   /* clusters                                            */
    int nb_max;       /* largest number of 16-row blocks of one row group    */
    int k_slice;      /* K columns per CTA of a cluster                      */
    long long smem_bytes; /* dynamic shared memory per CTA                   */
} wl_rows_plan;

/* Fills *out for the call on a GPU with num_sms SMs.  Returns
 * WL_ERR_UNSUPPORTED for calls the row-stream kernel does not take, and the
 * argument errors of wl_stacked_forward. */
wl_status wl_describe_rows_plan(int M, int K, const wl_proj *projs, int P, int num_sms,
                                wl_rows_plan *out);

/* Static description of a status code. */
const char *wl_status_string(wl_status status);

/* Synchronises `stream`, then returns and clears the current device's status
 * word: WL_OK, or the first error a kernel recorded since the last call (for
 * example WL_ERR_TIMEOUT from a wait that gave up). */
wl_status wl_last_device_status(void *stream);

/* Sets the time limit of every device-side wait of the forward calls issued
 * afterwards, on every device (limit_ns in nanoseconds, 1 ..  1e10; 0 restores
 * the default of 2 s).  For tests of the time-out path: a short limit makes
 * waits give up (WL_ERR_TIMEOUT via wl_last_device_status) instead of
 * waiting; every wait is bounded either way.  Returns WL_ERR_INVALID_ARG
 * outside that range. */
wl_status wl_set_wait_limit(long long limit_ns);

/* Launches one probe kernel that waits on a device flag nothing ever sets,
 * giving up after `limit_ns` nanoseconds and recording WL_ERR_TIMEOUT in the
 * device status word, exactly as the forward kernels do when one of their
 * waits expires.  Lets tests check the time-out path without a hung GPU.
 * 0 < limit_ns <= 1e9.  Asynchronous on `stream`. */
wl_status wl_wait_probe(long long limit_ns, void *stream);

/* Library version, (major << 16) | minor. */
int wl_version(void);

#ifdef __cplusplus
}
#endif

#endif /* WL_H_ */
