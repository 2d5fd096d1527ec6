/*
 * libmoe -- one mixture-of-experts feed-forward layer, forward and backward,
 * on one NVIDIA B200 (sm_100a).  Plain C ABI: pointers, sizes, a CUDA stream.
 *
 * Passages cited below (page title, section):
 *  [OC3-ja]  "Olmo-core 3 オープン混合エキスパート学習インフラストラクチャ"
 *            (agentlenshq.com), section "ルーティングと計算の最適化": routed
 *            tokens are written directly into the experts' input buffers
 *            ("rowwise" dispatch), routing metadata stays on the GPU so the
 *            CPU is never a bottleneck, and many small per-expert matmuls are
 *            batched into one grouped GEMM.  Section "MXFP8による精度最適化":
 *            MXFP8 as the low-precision format of the expert feed-forward
 *            compute.  Section "実証されたスケール": random routing used to
 *            stress the system.
 *  [OC3-hu]  "Az Ai2 megnyitotta az Olmo-core 3 MoE-tréningrendszerét"
 *            (aihirek.info), first section: 8 -> 128 experts with four chosen
 *            per token; section "Billió paraméteres tesztek, nyílt
 *            hozzáférés": rowwise dispatch, GPU-resident routing, grouped GEMM.
 *  [OC3-th]  "เปิดตัว Olmo-core 3 ..." (ai4bro.com), section on scaling and
 *            optimising MoE training: GPU-resident routing lets the CPU queue
 *            work without waiting for copies.
 *  [JUPITER] "PyTorch、欧州の公共スパコンで約1兆パラメータMoEを訓練"
 *            (cctest.ai), model paragraph: 384 experts, top-8, hidden 6144.
 *
 * The layer (its formulas are not printed on the pages; this is the layer
 * definition the library implements):
 *   logits  L = x W_r (+ b)                       x [T,d] bf16, W_r [d,E] fp32
 *   top-k   k largest logits per token, ties -> lower expert index
 *   gates   softmax over the k chosen logits (= softmax over E, renormalised)
 *   expert  y_e(x) = (silu(x W1[e]) * (x W3[e])) W2[e]
 *   out[t]  = sum_j gates[t,j] * y_{topk[t,j]}(x[t])
 *
 * Conventions for every call:
 *  - Asynchronous and stream-ordered on `stream`; never synchronises the
 *    host, never allocates device memory.  The caller owns every buffer.
 *  - Device pointers unless stated otherwise; 16-byte aligned.
 *  - bf16 arrays are passed as `void*` (IEEE bfloat16 bit patterns).
 *  - All matrices row-major.  Weight layout: W1, W3 [E,d,F]; W2 [E,F,d];
 *    W_r [d,E].
 *  - Returns MOE_OK, or an error code with nothing enqueued (argument
 *    errors) or after a failed launch (MOE_ERR_CUDA).  moe_last_error()
 *    gives a message for the calling thread.
 *  - Data errors found on the device (an expert index out of range, a
 *    duplicate expert in a token, a pipeline wait that gave up) are OR-ed
 *    into the caller's `int32_t* dev_status` word (MOE_DEV_* bits; may be
 *    NULL), which the caller reads whenever it chooses.  No kernel traps.
 *
 * Routing metadata (bit-exact, GPU resident):
 *   counts[E]     assignments per expert
 *   offsets[E+1]  exclusive scan of counts
 *   poff[E+1]     exclusive scan of counts rounded up to `align` (= 128):
 *                 group e occupies rows [poff[e], poff[e+1]) of every
 *                 expert-contiguous buffer; its first counts[e] rows are real,
 *                 the rest are zero pad rows
 *   dst[T,k]      permuted row of assignment (t,j) =
 *                 poff[e] + #{t' < t : expert e chosen by t'}  (stable)
 *   src[A_pad_max] token of each permuted row, -1 for pad rows
 *   A_pad_max     = T*k + E*(align-1), the host-known bound on poff[E]
 *
 * MX (MXFP8) tensors: codes are E4M3FN bytes with the shape of the source;
 * one E8M0 scale byte per 32 elements along the GEMM's K axis, with
 * X = 2^(floor(log2 amax) - 8), round-to-nearest-even, saturation at 448;
 * an all-zero block gets byte 0.  Scales are stored in the tensor-core
 * layout: for a source [R, C] quantised along axis a (a = 0: blocks along a
 * row, K = C, MN = R; a = 1: blocks down a column, K = R, MN = C), the scale
 * of (mn, kb) (kb = K index / 32) sits at byte
 *   ((mn/128) * (K/128) + kb/4) * 512 + (mn%32)*16 + ((mn/32)%4)*4 + kb%4.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* a cudaStream_t (NULL = legacy default) */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* a size, pointer, alignment or mode is not accepted */
  MOE_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement */
  MOE_ERR_WORKSPACE = 3,    /* workspace / context smaller than the query says */
  MOE_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed */
  MOE_ERR_TIMEOUT = 5,      /* reserved: host-visible form of MOE_DEV_TIMEOUT */
  MOE_ERR_DEVICE_DATA = 6   /* reserved: host-visible form of the MOE_DEV_* data bits */
} moe_status_t;

/* bits OR-ed into *dev_status by kernels */
#define MOE_DEV_BAD_EXPERT 0x1  /* a given expert index is outside [0, E) */
#define MOE_DEV_DUP_EXPERT 0x2  /* a token lists the same expert twice */
#define MOE_DEV_TIMEOUT 0x4     /* a GEMM pipeline wait gave up (bounded spin) */
#define MOE_DEV_NONFINITE 0x8   /* a router logit was NaN or infinite */

typedef enum { MOE_ROUTE_ROUTER = 0, MOE_ROUTE_GIVEN = 1 } moe_route_mode;
typedef enum { MOE_BF16 = 0, MOE_MXFP8 = 1 } moe_dtype;
typedef enum {
  MOE_EPI_NONE = 0,       /* C = A B */
  MOE_EPI_SWIGLU = 1,     /* fwd GEMM1: C = silu(A W1) * (A W3), aux = [A W1 | A W3] */
  MOE_EPI_SWIGLU_BWD = 2  /* dgrad of GEMM2 fused with the SwiGLU backward */
} moe_epilogue;

/* Message for the last failed call on this thread ("" if none). */
MOE_API const char* moe_last_error(void);
/* Library version string. */
MOE_API const char* moe_version(void);
/* Number of kernels this library has launched in this process. */
MOE_API unsigned long long moe_launch_count(void);

/* Benchmark hook: when set (per host thread), moe_layer_fwd / moe_layer_bwd
 * record events[2*s] before and events[2*s+1] after stage s on the stream
 * (cudaEvent_t handles; n = number of handles; NULL disables).  Stages:
 *   0 route  1 permute  2 quantise fwd weights  3 GEMM1+SwiGLU  4 quantise h
 *   5 GEMM2  6 combine  7 combine bwd  8 quantise for GEMM2 dgrad
 *   9 GEMM2 dgrad+SwiGLU bwd  10 quantise for GEMM2 wgrad  11 GEMM2 wgrad
 *   12 quantise for GEMM1 dgrad  13 GEMM1 dgrad  14 quantise for GEMM1 wgrad
 *   15 GEMM1 wgrad  16 unpermute-sum  17 router weight grad
 * (quantise stages run in MXFP8 mode only). */
#define MOE_NUM_STAGES 18
MOE_API void moe_set_stage_events(void* const* events, int n);

/* ------------------------------------------------------------------ route
 * Router and GPU-resident routing metadata ([OC3-ja] "ルーティングと計算の最適化":
 * metadata kept on the GPU; [OC3-th]: the CPU queues work without waiting
 * for copies; [OC3-hu] first section / [JUPITER]: k experts per token).
 *
 * mode MOE_ROUTE_ROUTER: logits = x W_r (+ bias) in fp32, top-k (ties to the
 *   lower index, slot j = j-th largest), gates = softmax of the k chosen
 *   logits (fp32); writes topk_idx [T,k] and gates [T,k].  With E <= 128,
 *   E % 8 == 0, k <= 8 and d % 64 == 0 the logits run on the tensor cores:
 *   W_r is split into two bf16 parts (w0 + w1 = W_r within 2^-17 |W_r|,
 *   below the fp32 accumulation error of a sum over d >= 32 terms; each
 *   product exact) accumulated in fp32; otherwise fp32 FMA on CUDA cores.
 * mode MOE_ROUTE_GIVEN: topk_idx and gates are INPUTS (random-routing stress
 *   workload, [OC3-ja] "実証されたスケール"); x and W_r are not read.  An index
 *   outside [0,E) or a repeat inside a token sets MOE_DEV_BAD_EXPERT /
 *   MOE_DEV_DUP_EXPERT and that assignment is dropped (dst = -1).
 * Both modes then write counts, offsets, poff, dst and src (see above).
 *   logits: optional [T,E] fp32 copy of the router logits (ROUTER mode).
 *   align must be 128.  Router mode needs E <= 512, k <= min(E, 16),
 *   d % 8 == 0; given mode E <= 4096.
 *   ws: 256-byte aligned device workspace of at least
 *   moe_route_workspace_size(T, d, E) bytes (pass d = 0 for given mode).
 */
MOE_API size_t moe_route_workspace_size(int T, int d, int E);
MOE_API moe_status_t moe_route(const void* x, const float* Wr, const float* bias, int T, int d,
                       int E, int k, int align, int mode, int32_t* topk_idx, float* gates,
                       int32_t* counts, int32_t* offsets, int32_t* poff, int32_t* dst,
                       int32_t* src, int A_pad_max, float* logits, void* ws, size_t ws_bytes,
                       int32_t* dev_status, moe_stream_t stream);

/* moe_route_noalloc: moe_route with no workspace argument, for callers that
 * cannot allocate device memory while they run (a host whose device memory
 * is owned by a pooling allocator, or a latency-critical loop that must not
 * call cudaMalloc, which can synchronise the device and take an unbounded
 * time).  The pages have no counterpart to this call; it is a library
 * convenience.  Its scratch is a fixed, library-owned array in device memory
 * of MOE_ROUTE_NOALLOC_MAX_SCRATCH_BYTES (4 MiB) on every device that loads
 * the library, kept until the process exits; the caller still passes all
 * inputs and outputs.  Limit: moe_route_workspace_size(T, d, E) (d = 0 in
 * given mode) must fit, e.g. T = 65536, d = 2048, E = 128 in router mode or
 * T <= 262144 with E = 128 in given mode; larger sizes return
 * MOE_ERR_INVALID_ARG.  The first call on a device looks up the
 * array's device address (cudaGetSymbolAddress), so make that first call
 * before any stream capture.  All calls share the one array: calls that
 * overlap on the GPU (other streams, other host threads) race and must be
 * serialised by the caller.  Arguments and results as moe_route. */
#define MOE_ROUTE_NOALLOC_MAX_SCRATCH_BYTES (4u << 20)
MOE_API moe_status_t moe_route_noalloc(const void* x, const float* Wr, const float* bias, int T,
                                       int d, int E, int k, int align, int mode,
                                       int32_t* topk_idx, float* gates, int32_t* counts,
                                       int32_t* offsets, int32_t* poff, int32_t* dst,
                                       int32_t* src, int A_pad_max, float* logits,
                                       int32_t* dev_status, moe_stream_t stream);

/* ---------------------------------------------------------------- permute
 * Rowwise dispatch ([OC3-ja] "ルーティングと計算の最適化": routed tokens are
 * written directly into the experts' input buffers): Xp[dst[t,j]] = x[t]
 * for every assignment, and every pad row of every group is zeroed.
 *   x [T,d] bf16; Xp [A_pad_max,d] bf16; d % 8 == 0.
 *   Xq / Xs (both NULL or both set): additionally writes the MX codes of Xp
 *   [A_pad_max,d] and its scales along d (axis 0) -- MX requires d % 128 == 0.
 */
MOE_API moe_status_t moe_permute(const void* x, const int32_t* dst, const int32_t* offsets,
                         const int32_t* poff, int T, int k, int d, int E, int A_pad_max,
                         void* Xp, uint8_t* Xq, uint8_t* Xs, moe_stream_t stream);

/* ------------------------------------------------------------- mx_quantize
 * MX quantiser ([OC3-ja] "MXFP8による精度最適化"; rule in the file header).
 *   in [rows, cols] bf16.  axis 0: blocks of 32 along each row (K = cols);
 *   axis 1: blocks of 32 down each column (K = rows).  rows % 128 == 0 and
 *   cols % 128 == 0.  `poff` is accepted for documentation of grouped use:
 *   with axis 1 every group start must be a multiple of 128 (true for the
 *   routing metadata above), so no block crosses a group; it may be NULL.
 *   codes [rows, cols] u8; scales rows*cols/32 bytes in the layout above.
 *   `nrows_dev` (nullable device int): rows at and beyond *nrows_dev are
 *   skipped (their codes and scales are left as they are).
 */
MOE_API moe_status_t mx_quantize(const void* in, int rows, int cols, int axis, const int32_t* poff,
                         int E, const int32_t* nrows_dev, uint8_t* codes, uint8_t* scales,
                         moe_stream_t stream);

/* mx_quantize_dual: both quantisations of one bf16 [rows, cols] tensor from
 * a single pass -- codes_rows / scales_rows as mx_quantize axis 0 (blocks
 * along a row) and codes_cols / scales_cols as axis 1 (blocks down a
 * column), bit-identical to the two separate calls.  Every operand that
 * feeds two GEMMs with different K axes (weights, h, dY, dA13) needs both. */
MOE_API moe_status_t mx_quantize_dual(const void* in, int rows, int cols,
                                      const int32_t* nrows_dev, uint8_t* codes_rows,
                                      uint8_t* scales_rows, uint8_t* codes_cols,
                                      uint8_t* scales_cols, moe_stream_t stream);

/* ------------------------------------------------------- grouped GEMMs
 * Grouped GEMM over the expert groups of the routing metadata ([OC3-ja]
 * "ルーティングと計算の最適化": many small per-expert matmuls as one grouped
 * GEMM).  tcgen05 tensor cores, TMEM accumulators, TMA-fed shared-memory
 * pipeline, persistent CTAs walking a device-side tile schedule read from
 * poff (no host sync).  fp32 accumulation, bf16 outputs.
 *
 * Rows of group e are [poff[e], poff[e+1]); poff[E] <= A_pad_max; every
 * poff entry is a multiple of 128.  Shapes: K % 64 == 0 (BF16) or
 * K % 128 == 0 (MXFP8); N % 256 == 0 (N % 128 for SWIGLU halves).
 *
 * moe_grouped_gemm_fwd: for every row r of group e,
 *   EPI_NONE:   C[r, :N]  = A[r, :K] B[e]             B [E,K,N]
 *   EPI_SWIGLU: H1 = A[r] B[e], H3 = A[r] B3[e]        B, B3 [E,K,N], N = F
 *               C[r, :F] = silu(H1) * H3; aux (nullable) [A_pad_max, 2F]
 *               receives [H1 | H3] in bf16.
 *   dt == MOE_MXFP8: A, B, B3 are MX codes with scales A_sc (axis 0 of A),
 *   B_sc / B3_sc (axis 1 of the [E*K, N] view).
 */
MOE_API moe_status_t moe_grouped_gemm_fwd(int dt, const void* A, const uint8_t* A_sc, const void* B,
                                  const uint8_t* B_sc, const void* B3, const uint8_t* B3_sc,
                                  const int32_t* poff, int E, int A_pad_max, int N, int K,
                                  int epilogue, void* C, void* aux, int32_t* dev_status,
                                  moe_stream_t stream);

/* moe_grouped_gemm_dgrad: gradient through B[e] (B [E,K,N] as in fwd):
 *   EPI_NONE, B3 == NULL: dA[r, :K] = dC[r, :N] B[e]^T
 *   EPI_NONE, B3 != NULL: dC has 2N columns; dA = dC[:, :N] B[e]^T + dC[:, N:] B3[e]^T
 *   EPI_SWIGLU_BWD (B = W2 [E,F,d], so K = F, N = d): dh = dC B[e]^T and,
 *     with aux = [H1 | H3] [A_pad_max, 2F] from the forward,
 *     dA[r, :F]  = dh * H3 * s * (1 + H1 (1 - s)),  s = sigmoid(H1)
 *     dA[r, F:]  = dh * silu(H1)                     (dA is [A_pad_max, 2F])
 *   dt == MOE_MXFP8: dC codes with dC_sc along its columns (axis 0); B / B3
 *   codes with scales along N, i.e. axis 0 of the [E*K, N] view.
 */
MOE_API moe_status_t moe_grouped_gemm_dgrad(int dt, const void* dC, const uint8_t* dC_sc,
                                    const void* B, const uint8_t* B_sc, const void* B3,
                                    const uint8_t* B3_sc, const int32_t* poff, int E,
                                    int A_pad_max, int N, int K, int epilogue, const void* aux,
                                    void* dA, int32_t* dev_status, moe_stream_t stream);

/* moe_grouped_gemm_wgrad: weight gradient, reduction over the rows of each
 * group:  dB[e][:K, :N] = A_e^T dC_e, A [A_pad_max, K], dC [A_pad_max, N].
 *   dB3 != NULL: dC has 2N columns; dB[e] = A_e^T dC_e[:, :N] and
 *   dB3[e] = A_e^T dC_e[:, N:].  Empty groups give zero gradients.
 *   Pad rows must be zero in A or dC (they are, for buffers written by this
 *   library).  dt == MOE_MXFP8: A and dC codes with scales down the columns
 *   (axis 1).
 */
MOE_API moe_status_t moe_grouped_gemm_wgrad(int dt, const void* A, const uint8_t* A_sc, const void* dC,
                                    const uint8_t* dC_sc, const int32_t* poff, int E,
                                    int A_pad_max, int K, int N, void* dB, void* dB3,
                                    int32_t* dev_status, moe_stream_t stream);

/* Rowwise dispatch straight into MX codes ([OC3-ja] "ルーティングと計算の最適化":
 * routed token rows go directly into the experts' input buffers; "MXFP8に
 * よる精度最適化").  Row r of the expert-contiguous buffer is token src[r]
 * (src from moe_route; -1 = a zero pad row); it is written only as MX codes,
 * along d (Xq [A_pad_max, d], Xs: scales along the row, K = d; the forward
 * GEMM1 operand) and down the rows in blocks of 32 inside each group (XqT
 * [A_pad_max, d], XsT: K = A_pad_max; the GEMM1 weight-gradient operand),
 * bit-identical to mx_quantize_dual of the bf16 permuted buffer.  No bf16
 * copy is written; rows from poff[E] on are not touched.  d % 128 == 0,
 * A_pad_max % 128 == 0, x / Xq / XqT 16-byte aligned. */
MOE_API moe_status_t moe_permute_mx(const void* x, const int32_t* src, const int32_t* poff,
                                    int T, int d, int E, int A_pad_max, uint8_t* Xq,
                                    uint8_t* Xs, uint8_t* XqT, uint8_t* XsT,
                                    moe_stream_t stream);

/* The backward's gate-scaled upstream rows straight into MX codes: row r of
 * the expert-contiguous buffer, in group e, is dY[r] = bf16(g * dout[t])
 * with t = src[r] and g = gates[t, j] for the slot j where topk_idx[t, j] =
 * e (a zero row for src[r] < 0), written only as MX codes along d (dYq /
 * dYs, K = d: GEMM2 dgrad) and down the rows (dYTq / dYTs, K = A_pad_max:
 * GEMM2 weight gradient); bit-identical to mx_quantize_dual of the dY that
 * moe_combine_bwd writes.  Rows from poff[E] on are not touched.  d % 128
 * == 0, k <= 16, E <= 1024. */
MOE_API moe_status_t moe_combine_bwd_mx(const void* dout, const float* gates,
                                        const int32_t* topk_idx, const int32_t* src,
                                        const int32_t* poff, int T, int k, int d, int E,
                                        int A_pad_max, uint8_t* dYq, uint8_t* dYs,
                                        uint8_t* dYTq, uint8_t* dYTs, moe_stream_t stream);

/* MXFP8 GEMMs whose SwiGLU epilogues quantise their bf16 result instead of
 * storing it ([OC3-ja] "MXFP8による精度最適化": the FP8 gain comes from
 * faster feed-forward compute and less data movement).  Each epilogue warp
 * owns a 32 x 32 block of the result, so both MX blocks of an element are
 * local: along the row (32 columns of one row) and down the column (32 rows
 * of one column, always inside one expert group).  Codes and scales are
 * bit-identical to mx_quantize_dual of the bf16 result the plain MX call
 * would store.  Scales in the tensor-core layout: along the row with K =
 * the row length, down the columns with K = A_pad_max.  Rows >= poff[E]
 * are not written.
 *   moe_grouped_gemm_fwd_swiglu_mxq: as moe_grouped_gemm_fwd(MOE_MXFP8,
 *     EPI_SWIGLU) with N = F; aux = [H1 | H3] bf16 (required); h -> h_q /
 *     h_s (along F) and hT_q / hT_s (down the rows).  F % 128 == 0.
 *   moe_grouped_gemm_dgrad_swiglu_mxq: as moe_grouped_gemm_dgrad(MOE_MXFP8,
 *     EPI_SWIGLU_BWD) with B = W2 codes along N = d, K = F; dA = [dA1 | dA3]
 *     [A_pad_max, 2F] -> dA_q / dA_s (along 2F) and dAT_q / dAT_s (down the
 *     rows).  K % 256 == 0. */
MOE_API moe_status_t moe_grouped_gemm_fwd_swiglu_mxq(
    const void* A, const uint8_t* A_sc, const void* B, const uint8_t* B_sc, const void* B3,
    const uint8_t* B3_sc, const int32_t* poff, int E, int A_pad_max, int F, int K, void* aux,
    uint8_t* h_q, uint8_t* h_s, uint8_t* hT_q, uint8_t* hT_s, int32_t* dev_status,
    moe_stream_t stream);
MOE_API moe_status_t moe_grouped_gemm_dgrad_swiglu_mxq(
    const void* dC, const uint8_t* dC_sc, const void* B, const uint8_t* B_sc,
    const int32_t* poff, int E, int A_pad_max, int N, int K, const void* aux, uint8_t* dA_q,
    uint8_t* dA_s, uint8_t* dAT_q, uint8_t* dAT_s, int32_t* dev_status, moe_stream_t stream);

/* Dispatch fused into the GEMM ([OC3-ja] "ルーティングと計算の最適化": routed
 * token rows go straight into the experts' input; here they go straight into
 * the GEMM's shared-memory tiles).  BF16 only.  Same products as
 * moe_grouped_gemm_fwd / moe_grouped_gemm_wgrad on the permuted buffer Xp,
 * but row r of that operand is read from the unpermuted tokens x [T, K]
 * as x[src[r]] (src from moe_route: the token of each padded row, -1 for a
 * pad row, which reads as zeros), by TMA row gathers in the GEMM's
 * producer; Xp is never written.  x and src 16-byte aligned; K % 64 == 0
 * (fwd) or K % 128 == 0 (wgrad); the weight and dC maps must be 3-D (the
 * library's layout; otherwise MOE_ERR_INVALID_ARG).
 *   moe_grouped_gemm_fwd_gather:   epilogue NONE or SWIGLU as in
 *     moe_grouped_gemm_fwd, with A = x gathered.
 *   moe_grouped_gemm_wgrad_gather: dB[e] = Xp_e^T dC_e (dB3 as in
 *     moe_grouped_gemm_wgrad); `offsets` (the unpadded group offsets, or
 *     NULL) stops each group's reduction after its last real row. */
MOE_API moe_status_t moe_grouped_gemm_fwd_gather(const void* x, int T, const int32_t* src,
                                                 const void* B, const void* B3,
                                                 const int32_t* poff, int E, int A_pad_max,
                                                 int N, int K, int epilogue, void* C, void* aux,
                                                 int32_t* dev_status, moe_stream_t stream);
MOE_API moe_status_t moe_grouped_gemm_wgrad_gather(const void* x, int T, const int32_t* src,
                                                   const void* dC, const int32_t* poff,
                                                   const int32_t* offsets, int E, int A_pad_max,
                                                   int K, int N, void* dB, void* dB3,
                                                   int32_t* dev_status, moe_stream_t stream);

/* Grouped GEMM with the tokens on the MMA's N side, BF16 (Olmo-core 3
 * オープン混合エキスパート学習インフラストラクチャ, "ルーティングと計算の最適化": the
 * expert matmuls as one grouped GEMM).  The weights form the 128-row M side
 * of each tile; group e's real rows (offsets[e+1] - offsets[e], or all of
 * its padded rows when offsets is NULL) are split evenly into token blocks
 * of at most 256 (multiples of 32) on the N side, so padding rows are not
 * multiplied; output rows from the last real row to poff[e+1] are written
 * as zeros.  Same results as moe_grouped_gemm_fwd / _dgrad (BF16) up to
 * rounding, except that in the SwiGLU form h uses the bf16-rounded X W3.
 *   epilogue MOE_EPI_SWIGLU: X [A_pad_max, K], W and W3 [E, K, N] (N % 64
 *     == 0) -> C = h [A_pad_max, N], aux = [X W | X W3] [A_pad_max, 2N].
 *   MOE_EPI_NONE, w_kmajor = 0: C = X W, W [E, K, N], W3 NULL (N % 128).
 *   MOE_EPI_NONE, w_kmajor = 1: W (and W3) [E, N, Kw], K = Kw (W3 NULL) or
 *     2 Kw: C = X[:, :Kw] W^T (+ X[:, Kw:] W3^T), plus, when row_scale and
 *     col_vec are given, row_scale[row] * col_vec[e * N + n] (fp32,
 *     col_vec 16-byte aligned).  N % 128 == 0.
 * K % 64 == 0; E <= 1024; A_pad_max % 128 == 0.  Pointers are device
 * memory owned by the caller; returns MOE_ERR_INVALID_ARG on bad shapes. */
MOE_API moe_status_t moe_grouped_gemm_tn(int epilogue, const void* X, const void* W,
                                         const void* W3, int w_kmajor, const int32_t* poff,
                                         const int32_t* offsets, int E, int A_pad_max, int N,
                                         int K, void* C, void* aux, const float* row_scale,
                                         const float* col_vec, int32_t* dev_status,
                                         moe_stream_t stream);

/* Self-test of the failure detection the grouped GEMM relies on: a kernel
 * waits on an mbarrier that nothing arrives at, gives up after limit_ns
 * (at most 2 s), ORs MOE_DEV_TIMEOUT into *dev_status and returns, leaving
 * the context usable.  The GEMM's own waits use the same bounded wait (2 s):
 * a time-out there makes every role of the CTA drain its copies in flight,
 * release TMEM and exit, with MOE_DEV_TIMEOUT set. */
MOE_API moe_status_t moe_selftest_wait_timeout(int32_t* dev_status, uint64_t limit_ns,
                                               moe_stream_t stream);

/* -------------------------------------------------- unpermute / combine
 * Gate-weighted combine (the unpermute half of the rowwise dispatch of
 * [OC3-ja]): out[t] = sum_{j<k} gates[t,j] * Y[dst[t,j]], fp32 sum in slot
 * order, bf16 result.  gates == NULL gives the plain sum.  dst entries < 0
 * contribute nothing.  d % 8 == 0.
 */
MOE_API moe_status_t moe_unpermute_combine(const void* Y, const float* gates, const int32_t* dst,
                                   int T, int k, int d, void* out, moe_stream_t stream);

/* Backward of the combine: for each assignment (t,j) with r = dst[t,j]
 *   dY[r]    = bf16(gates[t,j] * dout[t]);  pad rows of dY are zeroed
 *              (dY nullable: then only dg / dl / dl_rows are written)
 *   dg[t,j]  = <dout[t], Y[r]>  (fp32)
 *   and, when dl != NULL (router mode), the logit gradient of the chosen
 *   experts dl[t,j] = g_j (dg_j - sum_i g_i dg_i) (fp32), also scattered to
 *   dl_rows[r] (nullable, [A_pad_max] fp32, pad rows of each group set to 0).
 */
MOE_API moe_status_t moe_combine_bwd(const void* dout, const void* Y, const float* gates,
                             const int32_t* dst, const int32_t* offsets, const int32_t* poff,
                             int T, int k, int d, int E, void* dY, float* dg, float* dl,
                             float* dl_rows, moe_stream_t stream);

/* Backward of the dispatch: dx[t] = sum_j dXp[dst[t,j]]
 *   (+ sum_j dl[t,j] W_r[:, topk_idx[t,j]] when Wr != NULL: the router's
 *   input gradient), fp32 sum, bf16 result.  ws: at least
 *   moe_unpermute_sum_workspace_size(d, E) bytes (a transposed W_r).
 */
MOE_API size_t moe_unpermute_sum_workspace_size(int d, int E);
MOE_API moe_status_t moe_unpermute_sum(const void* dXp, const int32_t* dst, const int32_t* topk_idx,
                               const float* dl, const float* Wr, int T, int k, int d, int E,
                               void* dx, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Router weight gradient: dWr[i, e] = sum over the real rows r of group e
 * of x[src[r], i] * dl_rows[r]  (= x^T dL with dL nonzero only at the chosen
 * experts), fp32 [d, E].  Reduced per 128-row block of the permuted buffer,
 * then per expert (fixed order, independent of the load skew).  ws: at
 * least moe_router_wgrad_workspace_size(d, A_pad_max) bytes.  `offsets` is
 * unused (kept for the call's symmetry with the other metadata users).
 */
MOE_API size_t moe_router_wgrad_workspace_size(int d, int A_pad_max);
MOE_API moe_status_t moe_router_wgrad(const void* x, const int32_t* src, const float* dl_rows,
                                      const int32_t* offsets, const int32_t* poff, int T, int d,
                                      int E, int A_pad_max, float* dWr, void* ws,
                                      size_t ws_bytes, moe_stream_t stream);

/* --------------------------------------------------------------- layer
 * The whole layer: route -> permute -> GEMM1+SwiGLU -> GEMM2 -> combine, and
 * its backward, on `stream`, with no host synchronisation and no device
 * allocation.  ([OC3-ja] "ルーティングと計算の最適化": the steps of one MoE
 * layer -- route, keep the metadata on the GPU, write the rows into the
 * experts' buffers, grouped GEMM, combine; "MXFP8による精度最適化": the
 * expert GEMMs in MXFP8 when desc.dtype is MOE_MXFP8; [OC3-hu] first
 * section and [JUPITER] model paragraph: the layer shapes, 128 experts with
 * 4 chosen per token, 384 with 8.)  All saved tensors live in the caller's context buffer `ctx`
 * of at least moe_layer_ctx_bytes(desc) bytes (256-byte aligned).  BF16
 * layers whose experts average fewer than 256 rows (T k < 256 E) run the
 * forward GEMMs and the GEMM1 dgrad on the tokens-N kernel
 * (moe_grouped_gemm_tn) with the unpadded group offsets; the others on
 * moe_grouped_gemm_fwd / _dgrad.  Either way every padded row of the saved
 * tensors is zero.
 */
typedef struct {
  int T, d, E, k, F;
  int align;       /* must be 128 */
  int route_mode;  /* moe_route_mode */
  int dtype;       /* moe_dtype of the grouped GEMMs */
} moe_layer_desc;

typedef struct {
  const float* Wr;         /* [d,E] fp32 (router mode) */
  const float* bias;       /* [E] fp32, nullable (router mode, constant) */
  const void* W1;          /* [E,d,F] bf16 */
  const void* W3;          /* [E,d,F] bf16 */
  const void* W2;          /* [E,F,d] bf16 */
  const int32_t* topk_idx; /* [T,k], given mode */
  const float* gates;      /* [T,k], given mode */
} moe_layer_weights;

typedef struct {
  void* dW1;   /* [E,d,F] bf16 */
  void* dW3;   /* [E,d,F] bf16 */
  void* dW2;   /* [E,F,d] bf16 */
  float* dWr;  /* [d,E] fp32 (router mode; nullable) */
} moe_layer_grads;

/* Pointers into a context buffer (for inspection and tests). */
typedef struct {
  int32_t *topk_idx, *counts, *offsets, *poff, *dst, *src;
  float *gates, *logits, *dg, *dl, *dl_rows;
  void *Xp, *H13, *h, *Y, *dY, *dA13, *dXp;        /* bf16 */
  uint8_t *Xp_q, *Xp_s, *W13_q, *W13_s, *W2_q, *W2_s, *h_q, *h_s;  /* MX (fwd) */
  uint8_t *dY_q, *dY_s, *W13t_q, *W13t_s, *W2t_q, *W2t_s, *dA_q, *dA_s;  /* MX (bwd) */
  uint8_t *hT_q, *hT_s, *dYT_q, *dYT_s, *XpT_q, *XpT_s, *dAT_q, *dAT_s;  /* MX (wgrad) */
  void* ws;
  size_t ws_bytes;
  int A_pad_max;
} moe_ctx_view;

/* Bytes of the context buffer the layer needs (host-side, no GPU work; 0
 * for a description the layer rejects).  The context holds what the
 * backward reuses from the forward ([OC3-ja] "ルーティングと計算の最適化":
 * routing metadata and expert buffers stay on the GPU). */
MOE_API size_t moe_layer_ctx_bytes(const moe_layer_desc* desc);
MOE_API moe_status_t moe_layer_ctx_view(const moe_layer_desc* desc, void* ctx, moe_ctx_view* view);

/* Forward of the layer: out [T,d] bf16 from x [T,d] bf16; saves into ctx
 * what the backward needs.  (Passages: as for the layer above.) */
MOE_API moe_status_t moe_layer_fwd(const moe_layer_desc* desc, const moe_layer_weights* w,
                           const void* x, void* out, void* ctx, size_t ctx_bytes,
                           int32_t* dev_status, moe_stream_t stream);

/* Backward of the layer (after moe_layer_fwd on the same ctx): dx and the
 * weight gradients.  In router mode the router's share of dx,
 * sum_j dl[t,j] W_r[:, topk_idx[t,j]], is added to each permuted row of dXp
 * by the GEMM1 dgrad epilogue (W_r^T staged in the ctx workspace), so dx is
 * the plain sum of the k rows of dXp of each token. */
MOE_API moe_status_t moe_layer_bwd(const moe_layer_desc* desc, const moe_layer_weights* w,
                           const void* x, void* ctx, size_t ctx_bytes, const void* dout,
                           void* dx, moe_layer_grads* grads, int32_t* dev_status,
                           moe_stream_t stream);

/* One training step of the layer from HOST buffers: copies x and dout
 * (pinned host memory recommended) to the device buffers x_dev / dout_dev,
 * runs moe_layer_fwd and moe_layer_bwd, and copies out and dx back to
 * out_host / dx_host.  The copies run on two streams the library creates
 * once per device (non-blocking, kept until exit), one for uploads and one
 * for downloads, ordered with events: out moves to the host under the
 * backward, and dx under the backward's last weight gradients (the backward
 * forms dx before them).  Each device buffer is ordered only against the
 * earlier host-buffer step that used it (the library keeps one event per
 * buffer for the last 32 buffers): an upload into x_dev / dout_dev waits
 * for that step's backward, and the forward / backward rewrite out_dev /
 * dx_dev only after that step's downloads; a buffer the library has not
 * seen waits for the work already on `stream`.  `stream` itself never waits
 * for the downloads, so a caller that alternates two sets of device buffers
 * gets each step's uploads under the previous step's backward and its
 * forward under the previous step's downloads.  Write the device buffers
 * only through this call.  The call returns once the work is enqueued; the
 * host outputs (and the reads of the host inputs) are complete after
 * moe_layer_step_host_sync(stream) and a synchronisation of `stream` (or of
 * the device).  It creates four CUDA events per call and keeps four; it
 * allocates no device memory.
 * ([OC3-th] scaling/optimisation section: the host queues the work without
 * waiting for copies.)
 */
MOE_API moe_status_t moe_layer_step_host(const moe_layer_desc* desc, const moe_layer_weights* w,
                                 const void* x_host, const void* dout_host, void* out_host,
                                 void* dx_host, void* x_dev, void* dout_dev, void* out_dev,
                                 void* dx_dev, void* ctx, size_t ctx_bytes,
                                 moe_layer_grads* grads, int32_t* dev_status,
                                 moe_stream_t stream);

/* Makes `stream` wait for every download moe_layer_step_host has queued on
 * the current device so far: after it, synchronising `stream` leaves every
 * earlier step's host outputs complete.  Enqueues only; returns
 * MOE_ERR_CUDA if the library's copy streams cannot be made or ordered.
 * (No counterpart in the pages: the host-side half of the asynchronous
 * step above.) */
MOE_API moe_status_t moe_layer_step_host_sync(moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
