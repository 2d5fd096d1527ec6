// Router (logits, top-k, gates) and GPU-resident routing metadata.
//
// Olmo-core 3 オープン混合エキスパート学習インフラストラクチャ, section
// "ルーティングと計算の最適化": routing metadata is kept on the GPU so the CPU
// never waits for it.  Nothing here copies to the host or synchronises.
//
// Three launches, all stream-ordered:
//   1. per block of tokens, the k experts of each token (router: fp32
//      logits, top-k, gates), each assignment's rank among the block's
//      assignments to the same expert (token order), and the block's
//      per-expert histogram.  Router mode runs on the tensor cores when it
//      can (E <= 128, E % 8 == 0, k <= 8, d % 64 == 0; blocks of 128 tokens):
//      W_r is split into two bf16 parts w0 + w1 (equal to W_r within
//      2^-17 |W_r|, below the fp32 accumulation error of a length-d sum for
//      d >= 32) and the logits are one K = 2d product [x|x] [w0;w1]
//      accumulated in fp32.  The
//      fallback (and given-mode) kernels use blocks of 32 tokens and fp32
//      FMA.
//   2. route_scan (one CTA): per-expert exclusive scan of the block
//      histograms -> block offsets, counts, offsets, padded offsets poff.
//   3. route_scatter: dst = poff[e] + block offset + in-block rank, src, and
//      -1 for every pad row.
// The result is the stable counting sort of the assignments by expert.
#include <mutex>

#include "common.cuh"

namespace moe {

constexpr int kTok = 32;        // tokens per routing block
constexpr int kRouteThreads = 256;
constexpr int kMaxRouterE = 512;
constexpr int kMaxK = 16;
constexpr int kKC = 32;         // d-chunk of the logit product
constexpr int kEC = 128;        // expert chunk of the logit product

// ---------------------------------------------------------------------------
// in-block ranks + histogram (shared by both modes).  sel[t][j] holds the
// expert of assignment (t,j) or -1 for a dropped one.
__device__ void block_rank_and_hist(const int* sel, int ntok, int k, int E, int* cnt,
                                    int32_t* rank_out /* dst, [T,k] */, int tok0,
                                    int32_t* hist_row /* [E] */) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    for (int t = 0; t < ntok; ++t) {
      int r = -1;
      if (lane < k) {
        int e = sel[t * k + lane];
        if (e >= 0) {       // the k experts of one token are distinct
          r = cnt[e];
          cnt[e] = r + 1;
        }
        rank_out[(size_t)(tok0 + t) * k + lane] = r;
      }
      __syncwarp();
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist_row[e] = cnt[e];
}

// ---------------------------------------------------------------------------
// Router mode.  Logits: fp32 FMA, d ascending, one accumulator per (t,e).
__global__ void __launch_bounds__(kRouteThreads)
route_topk_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ Wr,
                  const float* __restrict__ bias, int T, int d, int E, int k,
                  int32_t* __restrict__ topk_idx, float* __restrict__ gates,
                  float* __restrict__ logits_out, int32_t* __restrict__ rank_out,
                  int32_t* __restrict__ hist, int32_t* __restrict__ status) {
  __shared__ __align__(16) float xs[kKC][kTok];
  __shared__ __align__(16) float wsh[kKC][kEC];
  extern __shared__ float Ldyn[];   // [kTok][E + 1] logits of the block
  __shared__ int sel[kTok * kMaxK];
  __shared__ int cnt[kMaxRouterE];

  const int tid = threadIdx.x;
  const int tok0 = blockIdx.x * kTok;
  const int ntok = min(kTok, T - tok0);
  const int tx = tid & 31, ty = tid >> 5;

  for (int e0 = 0; e0 < E; e0 += kEC) {
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < d; k0 += kKC) {
      {  // x tile: 32 tokens x 32 columns, 4 bf16 per thread, stored transposed
        const int t = tid >> 3, c = (tid & 7) * 4;
        float v[4] = {0.f, 0.f, 0.f, 0.f};
        if (t < ntok && k0 + c < d) {   // d % 8 == 0 so 4-groups never straddle d
          const uint2 raw = *reinterpret_cast<const uint2*>(x + (size_t)(tok0 + t) * d + k0 + c);
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
          float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
          v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) xs[c + i][t] = v[i];
      }
      // W_r tile: 32 rows x 128 experts
#pragma unroll
      for (int i = 0; i < (kKC * kEC) / kRouteThreads; ++i) {
        const int idx = tid + i * kRouteThreads;
        const int r = idx / kEC, c = idx % kEC;
        float w = 0.f;
        if (k0 + r < d && e0 + c < E) w = Wr[(size_t)(k0 + r) * E + e0 + c];
        wsh[r][c] = w;
      }
      __syncthreads();
#pragma unroll 8
      for (int kk = 0; kk < kKC; ++kk) {
        const float4 xv = *reinterpret_cast<const float4*>(&xs[kk][ty * 4]);
        const float4 wv = *reinterpret_cast<const float4*>(&wsh[kk][tx * 4]);
        const float xa[4] = {xv.x, xv.y, xv.z, xv.w};
        const float wa[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(xa[i], wa[j], acc[i][j]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int e = e0 + tx * 4 + j;
        if (e < E) Ldyn[(ty * 4 + i) * (E + 1) + e] = acc[i][j] + (bias ? bias[e] : 0.f);
      }
  }
  __syncthreads();

  // top-k per token: one warp per token, k rounds of a warp arg-max over
  // (value desc, index asc); NaN counts as -inf and is reported
  const int warp = tid >> 5, lane = tid & 31;
  for (int t = warp; t < ntok; t += kRouteThreads / 32) {
    uint32_t taken = 0;   // bit i: expert lane + 32 i already chosen
    float sv[kMaxK];
    int se[kMaxK];
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int be = 0x7fffffff;
      for (int i = 0; lane + 32 * i < E; ++i) {
        if (taken & (1u << i)) continue;
        float v = Ldyn[t * (E + 1) + lane + 32 * i];
        if (v != v) { v = -INFINITY; report(status, MOE_DEV_NONFINITE); }
        const int e = lane + 32 * i;
        if (v > bv || (v == bv && e < be)) { bv = v; be = e; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oe = __shfl_xor_sync(0xffffffffu, be, o);
        if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
      }
      if ((be & 31) == lane) taken |= 1u << (be >> 5);
      sv[j] = bv;
      se[j] = be;
    }
    // gates: softmax over the chosen logits (sv[0] is the largest)
    float s = 0.f;
    for (int j = 0; j < k; ++j) s += expf(sv[j] - sv[0]);
    for (int j = 0; j < k; ++j) {
      if (lane == j) {
        const size_t o = (size_t)(tok0 + t) * k + j;
        topk_idx[o] = se[j];
        gates[o] = expf(sv[j] - sv[0]) / s;
        sel[t * k + j] = se[j];
      }
    }
    if (logits_out)
      for (int e = lane; e < E; e += 32) logits_out[(size_t)(tok0 + t) * E + e] = Ldyn[t * (E + 1) + e];
  }
  __syncthreads();
  block_rank_and_hist(sel, ntok, k, E, cnt, rank_out, tok0, hist + (size_t)blockIdx.x * E);
}

// ---------------------------------------------------------------------------
// Given mode: validate the given experts; drop (and report) bad ones.
__global__ void __launch_bounds__(kRouteThreads)
route_given_kernel(const int32_t* __restrict__ topk_idx, int T, int E, int k,
                   int32_t* __restrict__ rank_out, int32_t* __restrict__ hist,
                   int32_t* __restrict__ status) {
  extern __shared__ int dyn[];
  int* cnt = dyn;              // [E]
  int* sel = dyn + E;          // [kTok * k]
  const int tok0 = blockIdx.x * kTok;
  const int ntok = min(kTok, T - tok0);
  for (int a = threadIdx.x; a < ntok * k; a += blockDim.x) {
    const int t = a / k, j = a % k;
    int e = topk_idx[(size_t)(tok0 + t) * k + j];
    if (e < 0 || e >= E) {
      report(status, MOE_DEV_BAD_EXPERT);
      e = -1;
    } else {
      for (int jj = 0; jj < j; ++jj)
        if (topk_idx[(size_t)(tok0 + t) * k + jj] == e) {
          report(status, MOE_DEV_DUP_EXPERT);
          e = -1;
          break;
        }
    }
    sel[a] = e;
  }
  __syncthreads();
  block_rank_and_hist(sel, ntok, k, E, cnt, rank_out, tok0, hist + (size_t)blockIdx.x * E);
}

// ---------------------------------------------------------------------------
// W_r [d, E] fp32 -> wsplit [2d, E] bf16 with w0 = bf16(W), w1 = bf16(W - w0):
// the difference is exact in fp32 and w0 + w1 keeps 16 significant bits, so
// |W - w0 - w1| <= 2^-17 |W| (normal range).
__global__ void router_split_kernel(const float* __restrict__ Wr, int n,
                                    __nv_bfloat16* __restrict__ ws) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float w = Wr[i];
  const __nv_bfloat16 w0 = __float2bfloat16_rn(w);
  ws[i] = w0;
  ws[n + i] = __float2bfloat16_rn(w - __bfloat162float(w0));
}

// ---------------------------------------------------------------------------
// One CTA: hist[b][e] -> exclusive offset of block b inside expert e;
// counts, offsets, poff.
constexpr int kScanThreads = 1024;
constexpr int kScanBatch = 8;

__global__ void __launch_bounds__(kScanThreads)
route_scan_kernel(int32_t* __restrict__ hist, int nblk, int E, int align,
                  int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                  int32_t* __restrict__ poff) {
  extern __shared__ int sm[];
  const int tid = threadIdx.x;
  // groups of blocks per expert so all threads work when E is small
  const int G = E <= kScanThreads ? max(1, kScanThreads / E) : 1;
  int* part = sm;                       // [G][E]  (G*E <= max(E, 1024))
  int* tot = sm + G * E;                // [E]
  const int chunk = (nblk + G - 1) / G;

  // the column of a (group, expert) work item is read kScanBatch blocks at
  // a time, all loads of a batch in flight together
  for (int w = tid; w < G * E; w += kScanThreads) {
    const int g = w / E, e = w % E;
    const int b0 = g * chunk, b1 = min(nblk, b0 + chunk);
    int s = 0;
    for (int b = b0; b < b1; b += kScanBatch) {
      int v[kScanBatch];
#pragma unroll
      for (int i = 0; i < kScanBatch; ++i) v[i] = b + i < b1 ? hist[(size_t)(b + i) * E + e] : 0;
#pragma unroll
      for (int i = 0; i < kScanBatch; ++i) s += v[i];
    }
    part[g * E + e] = s;
  }
  __syncthreads();
  for (int e = tid; e < E; e += kScanThreads) {
    int run = 0;
    for (int g = 0; g < G; ++g) {
      const int v = part[g * E + e];
      part[g * E + e] = run;
      run += v;
    }
    tot[e] = run;
    counts[e] = run;
  }
  __syncthreads();
  for (int w = tid; w < G * E; w += kScanThreads) {
    const int g = w / E, e = w % E;
    const int b0 = g * chunk, b1 = min(nblk, b0 + chunk);
    int run = part[g * E + e];
    for (int b = b0; b < b1; b += kScanBatch) {
      int v[kScanBatch];
#pragma unroll
      for (int i = 0; i < kScanBatch; ++i) v[i] = b + i < b1 ? hist[(size_t)(b + i) * E + e] : 0;
#pragma unroll
      for (int i = 0; i < kScanBatch; ++i) {
        if (b + i < b1) hist[(size_t)(b + i) * E + e] = run;
        run += v[i];
      }
    }
  }
  // exclusive scans over experts: serial within each thread's chunk, then
  // across the threads by shuffles within each warp and over the 32 warp
  // totals
  static_assert(kScanThreads == 32 * 32, "two-level shuffle scan");
  __shared__ int wc[32], wp[32];
  const int per = (E + kScanThreads - 1) / kScanThreads;
  const int e0 = tid * per, e1 = min(E, e0 + per);
  int c = 0, p = 0;
  for (int e = e0; e < e1; ++e) {
    c += tot[e];
    p += (tot[e] + align - 1) / align * align;
  }
  const int lane = tid & 31, wid = tid >> 5;
  int ci = c, pi = p;   // inclusive over the warp's threads
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, ci, o), b = __shfl_up_sync(0xffffffffu, pi, o);
    if (lane >= o) { ci += a; pi += b; }
  }
  if (lane == 31) { wc[wid] = ci; wp[wid] = pi; }
  __syncthreads();
  if (wid == 0) {
    int x = wc[lane], y = wp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, x, o), b = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) { x += a; y += b; }
    }
    wc[lane] = x;   // inclusive over the warps
    wp[lane] = y;
  }
  __syncthreads();
  ci += wid ? wc[wid - 1] : 0;
  pi += wid ? wp[wid - 1] : 0;
  int oc = ci - c, op = pi - p;   // exclusive: the sums of all earlier chunks
  for (int e = e0; e < e1; ++e) {
    offsets[e] = oc;
    poff[e] = op;
    oc += tot[e];
    op += (tot[e] + align - 1) / align * align;
  }
  if (tid == kScanThreads - 1) {
    offsets[E] = ci;
    poff[E] = pi;
  }
}

// ---------------------------------------------------------------------------
// dst / src.  Blocks [0, nA) handle assignments; the next E blocks mark the
// pad rows of one expert each; the last block marks [poff[E], A_pad_max).
__global__ void route_scatter_kernel(const int32_t* __restrict__ topk_idx,
                                     const int32_t* __restrict__ hist, int T, int E, int k,
                                     int btok,
                                     const int32_t* __restrict__ counts,
                                     const int32_t* __restrict__ poff,
                                     int32_t* __restrict__ dst, int32_t* __restrict__ src,
                                     int A_pad_max, int nA_blocks) {
  const int b = blockIdx.x;
  if (b < nA_blocks) {
    const int a = b * blockDim.x + threadIdx.x;
    if (a >= T * k) return;
    const int t = a / k;
    const int rank = dst[a];     // in-block rank written by the first launch
    const int e = topk_idx[a];
    if (rank < 0 || e < 0 || e >= E) {
      dst[a] = -1;
      return;
    }
    const int r = poff[e] + hist[(size_t)(t / btok) * E + e] + rank;
    dst[a] = r;
    src[r] = t;
  } else if (b < nA_blocks + E) {
    const int e = b - nA_blocks;
    for (int r = poff[e] + counts[e] + threadIdx.x; r < poff[e + 1]; r += blockDim.x) src[r] = -1;
  } else {
    for (int r = poff[E] + threadIdx.x; r < A_pad_max; r += blockDim.x) src[r] = -1;
  }
}

}  // namespace moe

using namespace moe;

static bool use_tensor_router(int d, int E, int k) {
  return E <= 128 && E % 8 == 0 && k <= 8 && d % 64 == 0;
}

extern "C" size_t moe_route_workspace_size(int T, int d, int E) {
  if (T <= 0 || E <= 0 || d < 0) return 0;
  // fallback / given mode: histograms of 32-token blocks
  const size_t simt = round_up((size_t)((T + kTok - 1) / kTok) * E * sizeof(int32_t), 256);
  // tensor-core router: histograms of 128-token blocks + the split W_r
  const size_t tc = round_up((size_t)((T + 127) / 128) * E * sizeof(int32_t), 256) +
                    round_up((size_t)2 * d * E * sizeof(__nv_bfloat16), 256);
  return simt > tc ? simt : tc;
}

extern "C" moe_status_t moe_route(const void* x, const float* Wr, const float* bias, int T,
                                  int d, int E, int k, int align, int mode, int32_t* topk_idx,
                                  float* gates, int32_t* counts, int32_t* offsets, int32_t* poff,
                                  int32_t* dst, int32_t* src, int A_pad_max, float* logits,
                                  void* ws, size_t ws_bytes, int32_t* dev_status,
                                  moe_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  MOE_CHECK_ARG(T > 0 && E > 0 && k > 0 && k <= E && k <= kMaxK, "moe_route: bad T/E/k");
  MOE_CHECK_ARG(align == 128, "moe_route: align must be 128");
  MOE_CHECK_ARG(A_pad_max >= T * k + E * (align - 1), "moe_route: A_pad_max below T*k+E*(align-1)");
  MOE_CHECK_ARG(topk_idx && gates && counts && offsets && poff && dst && src,
                "moe_route: null output");
  MOE_CHECK_ARG(mode == MOE_ROUTE_ROUTER || mode == MOE_ROUTE_GIVEN, "moe_route: bad mode");
  const size_t need = moe_route_workspace_size(T, mode == MOE_ROUTE_ROUTER ? d : 0, E);
  if (!ws || ws_bytes < need) {
    set_error("moe_route: workspace %zu < %zu bytes", ws_bytes, need);
    return MOE_ERR_WORKSPACE;
  }
  MOE_CHECK_ARG((reinterpret_cast<uintptr_t>(ws) & 255) == 0, "moe_route: workspace must be 256-byte aligned");
  int btok = kTok;
  int32_t* hist = static_cast<int32_t*>(ws);
  if (mode == MOE_ROUTE_ROUTER && use_tensor_router(d, E, k)) {
    MOE_CHECK_ARG(x && Wr && aligned16(x), "moe_route: router mode needs 16B-aligned x and Wr");
    btok = 128;
    const size_t hist_bytes = round_up((size_t)((T + 127) / 128) * E * sizeof(int32_t), 256);
    __nv_bfloat16* wsplit =
        reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(ws) + hist_bytes);
    const int n = d * E;
    router_split_kernel<<<(n + 255) / 256, 256, 0, s>>>(Wr, n, wsplit);
    MOE_CHECK_LAUNCH("router_split");
    MOE_TRY(router_tc(x, wsplit, bias, T, d, E, k, logits, topk_idx, gates, dst, hist,
                      dev_status, s));
  } else if (mode == MOE_ROUTE_ROUTER) {
    MOE_CHECK_ARG(x && Wr, "moe_route: router mode needs x and Wr");
    MOE_CHECK_ARG(E <= kMaxRouterE, "moe_route: router mode supports E <= %d", kMaxRouterE);
    MOE_CHECK_ARG(d > 0 && d % 8 == 0 && aligned16(x), "moe_route: d %% 8 and 16B-aligned x");
    const size_t smem = (size_t)kTok * (E + 1) * sizeof(float);
    MOE_TRY(set_smem_limit(reinterpret_cast<const void*>(route_topk_kernel),
                           (size_t)kTok * (kMaxRouterE + 1) * sizeof(float), "route_topk"));
    const int nblk = (T + kTok - 1) / kTok;
    route_topk_kernel<<<nblk, kRouteThreads, smem, s>>>(
        static_cast<const __nv_bfloat16*>(x), Wr, bias, T, d, E, k, topk_idx, gates, logits, dst,
        hist, dev_status);
    MOE_CHECK_LAUNCH("route_topk");
  } else {
    MOE_CHECK_ARG(E <= 4096, "moe_route: given mode supports E <= 4096");
    const size_t smem = (E + kTok * k) * sizeof(int);
    const int nblk = (T + kTok - 1) / kTok;
    route_given_kernel<<<nblk, kRouteThreads, smem, s>>>(topk_idx, T, E, k, dst, hist,
                                                         dev_status);
    MOE_CHECK_LAUNCH("route_given");
  }
  {
    const int nblk = (T + btok - 1) / btok;
    const int G = E <= kScanThreads ? max(1, kScanThreads / E) : 1;
    const size_t smem = ((size_t)G * E + E) * sizeof(int);
    route_scan_kernel<<<1, kScanThreads, smem, s>>>(hist, nblk, E, align, counts, offsets, poff);
    MOE_CHECK_LAUNCH("route_scan");
  }
  const int nA = (T * k + 255) / 256;
  route_scatter_kernel<<<nA + E + 1, 256, 0, s>>>(topk_idx, hist, T, E, k, btok, counts, poff,
                                                  dst, src, A_pad_max, nA);
  MOE_CHECK_LAUNCH("route_scatter");
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// Routing without any device allocation by the caller.
//
// Some callers cannot call cudaMalloc once they are running: a host whose
// device memory is owned by a pooling allocator, or a latency-critical loop
// that must not allocate (an allocation can synchronise the device and take
// an unbounded time).  This entry point gives them the router and routing
// metadata with the block-histogram scratch held in a fixed array that the
// library owns in device memory.  Inputs and outputs still come from the
// caller.
namespace {

constexpr size_t kNoAllocScratchBytes = MOE_ROUTE_NOALLOC_MAX_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// One copy per device that loads the library; held until the process exits.
static __device__ __align__(256) unsigned char g_route_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  The array's
// name is only a host-side stand-in, so the address is looked up once per
// device with cudaGetSymbolAddress.
moe_status_t scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    set_error("moe_route_noalloc: no usable current device");
    return MOE_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess || !p) {
      set_error("moe_route_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
      return MOE_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status_t moe_route_noalloc(const void* x, const float* Wr, const float* bias,
                                          int T, int d, int E, int k, int align, int mode,
                                          int32_t* topk_idx, float* gates, int32_t* counts,
                                          int32_t* offsets, int32_t* poff, int32_t* dst,
                                          int32_t* src, int A_pad_max, float* logits,
                                          int32_t* dev_status, moe_stream_t stream) {
  MOE_CHECK_ARG(T > 0 && E > 0, "moe_route_noalloc: bad T/E");
  const size_t need = moe_route_workspace_size(T, mode == MOE_ROUTE_ROUTER ? d : 0, E);
  MOE_CHECK_ARG(need <= kNoAllocScratchBytes,
                "moe_route_noalloc: needs %zu scratch bytes (moe_route_workspace_size) but the "
                "fixed array holds %zu; use moe_route with a caller workspace",
                need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  MOE_TRY(scratch_for_current_device(&scratch));
  // the histogram rows are fully written by the first launch before they are
  // read, so nothing in the shared array needs clearing between calls
  return moe_route(x, Wr, bias, T, d, E, k, align, mode, topk_idx, gates, counts, offsets, poff,
                   dst, src, A_pad_max, logits, scratch, kNoAllocScratchBytes, dev_status,
                   stream);
}
