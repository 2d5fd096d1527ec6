// MX (MXFP8) quantiser: E4M3 codes with one E8M0 scale per 32 elements.
//
// Olmo-core 3 オープン混合エキスパート学習インフラストラクチャ, section
// "MXFP8による精度最適化": MXFP8 for the expert feed-forward compute.  Rule
// (OCP MX): X = 2^(floor(log2 amax) - 8), code = RNE-saturating E4M3 of v/X,
// an all-zero block gets scale byte 0.
//
// For a bf16 block, floor(log2 amax) is the exponent field of amax minus
// 127, so the scale byte is max(expfield(amax) - 8, 0), and 1/X is the fp32
// number with exponent field 254 - byte (exact power-of-two scaling).
// Scales go to the tensor-core layout (see the library header).
#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "mx.cuh"
#include "sm100.cuh"

namespace moe {

__device__ __forceinline__ size_t sf_offset(int mn, int kb, int kchunks) {
  return mx_sf_offset(mn, kb, kchunks);
}
__device__ __forceinline__ uint32_t scale_byte(float amax) { return mx_scale_byte(amax); }
__device__ __forceinline__ float inv_scale(uint32_t byte) { return mx_inv_scale(byte); }
__device__ __forceinline__ uint2 encode8(const float* f, float inv) { return mx_encode8(f, inv); }

// ------------------------------------------- blocks along rows (axis 0)
// one warp per 256-column segment of one row; 4 lanes per 32-element block
__global__ void mx_quant_rows_kernel(const uint4* __restrict__ in, int rows, int cols,
                                     const int32_t* __restrict__ nrows_dev,
                                     uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const int segs = (cols + 255) / 256;
  const long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= (long long)rows * segs) return;
  const int row = (int)(w / segs), seg = (int)(w % segs);
  if (nrows_dev && row >= *nrows_dev) return;
  const int col = seg * 256 + lane * 8;
  const bool active = col < cols;
  float f[8];
  float amax = 0.f;
  if (active) {
    unpack8(in[((size_t)row * cols + col) / 8], f);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
  }
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  if (!active) return;
  const uint32_t b = scale_byte(amax);
  *reinterpret_cast<uint2*>(codes + (size_t)row * cols + col) = encode8(f, inv_scale(b));
  if ((lane & 3) == 0) scales[sf_offset(row, col / 32, cols / 128)] = (uint8_t)b;
}

// ------------------------------------------ blocks down columns (axis 1)
// one warp per (32-row block, 256-column segment); 8 columns per lane
__global__ void mx_quant_cols_kernel(const __nv_bfloat16* __restrict__ in, int rows, int cols,
                                     const int32_t* __restrict__ nrows_dev,
                                     uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const int segs = (cols + 255) / 256;
  const long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= (long long)(rows / 32) * segs) return;
  const int rb = (int)(w / segs), seg = (int)(w % segs);
  const int r0 = rb * 32;
  if (nrows_dev && r0 >= *nrows_dev) return;
  const int col = seg * 256 + lane * 8;
  if (col >= cols) return;
  float amax[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int r = 0; r < 32; ++r) {
    float f[8];
    unpack8(*reinterpret_cast<const uint4*>(in + (size_t)(r0 + r) * cols + col), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax[i] = fmaxf(amax[i], fabsf(f[i]));
  }
  uint32_t b[8];
  float inv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    b[i] = scale_byte(amax[i]);
    inv[i] = inv_scale(b[i]);
    scales[sf_offset(col + i, rb, rows / 128)] = (uint8_t)b[i];
  }
  for (int r = 0; r < 32; ++r) {
    float f[8];
    unpack8(*reinterpret_cast<const uint4*>(in + (size_t)(r0 + r) * cols + col), f);
    uint32_t wv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(
          make_float2(f[2 * i] * inv[2 * i], f[2 * i + 1] * inv[2 * i + 1]), __NV_SATFINITE,
          __NV_E4M3);
      wv[i] = (uint32_t)c;
    }
    *reinterpret_cast<uint2*>(codes + (size_t)(r0 + r) * cols + col) =
        make_uint2(wv[0] | (wv[1] << 16), wv[2] | (wv[3] << 16));
  }
}

// -------------------------------------------- both axes from one read
// Scale bytes are packed into the 4-byte words of the tensor-core layout
// (one word = 4 consecutive K blocks of one MN index): a column's word holds
// the four 32-row sub-blocks of a 128-row block, a row's word four
// consecutive 32-column blocks.

// One 128 x 128 bf16 tile in shared memory quantised along both axes by 8
// warps: warp w takes rows 16w..16w+15 (half of one 32-row MX column block;
// warps 2b and 2b+1 combine their column maxima through `camax`), two rows
// per step with 16 lanes of 8 columns each (a 32-column row block is 4
// lanes).  The first pass writes the row codes (16 lanes x 8 bytes = one
// 128-byte row segment) and keeps the raw rows in registers for the column
// codes of the second; the scale bytes are gathered in shared memory and
// leave as whole words of the tensor-core layouts.  `chunk(rl, c)` is the
// shared address of 16-byte chunk c (columns 8c..8c+7) of tile row rl.
// `gate` (nullable, by tile row): the rows are first replaced by the bf16
// product gate x row.  Rows at and beyond `nrows` are not written (their
// column blocks still see them; a 32-row block wholly beyond gets scale 0).
// Contains three __syncthreads: every thread of the CTA calls it.
template <class Chunk>
__device__ __forceinline__ void mx_tile_both_axes(
    Chunk chunk, const float* gate, int r0, int c0, int nrows, int cols, int col_kchunks,
    uint8_t* __restrict__ codes_r, uint8_t* __restrict__ scales_r, uint8_t* __restrict__ codes_c,
    uint8_t* __restrict__ scales_c, float (*camax)[128], uint8_t (*srow_s)[4],
    uint8_t (*scol_s)[4]) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = lane & 15, hrow = lane >> 4;
  const int rl0 = warp * 16;
  const int col = c0 + 8 * c;
  uint4 raw[8];
  float cm[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) cm[i] = 0.f;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int rl = rl0 + 2 * s + hrow;
    raw[s] = *reinterpret_cast<const uint4*>(chunk(rl, c));
    float f[8];
    unpack8(raw[s], f);
    if (gate) {
      const float g = gate[rl];
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] *= g;
      raw[s] = pack8(f);
      unpack8(raw[s], f);
    }
    float ra = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      cm[i] = fmaxf(cm[i], fabsf(f[i]));
      ra = fmaxf(ra, fabsf(f[i]));
    }
    ra = fmaxf(ra, __shfl_xor_sync(0xffffffffu, ra, 1));
    ra = fmaxf(ra, __shfl_xor_sync(0xffffffffu, ra, 2));
    const uint32_t br = mx_scale_byte(ra);
    const int row = r0 + rl;
    if (row < nrows)
      *reinterpret_cast<uint2*>(codes_r + (size_t)row * cols + col) = mx_encode8(f, mx_inv_scale(br));
    if ((c & 3) == 0) srow_s[rl][c >> 2] = (uint8_t)br;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) cm[i] = fmaxf(cm[i], __shfl_xor_sync(0xffffffffu, cm[i], 16));
  if (hrow == 0) {
    *reinterpret_cast<float4*>(&camax[warp][8 * c]) = make_float4(cm[0], cm[1], cm[2], cm[3]);
    *reinterpret_cast<float4*>(&camax[warp][8 * c + 4]) = make_float4(cm[4], cm[5], cm[6], cm[7]);
  }
  __syncthreads();
  const bool blk_live = r0 + (warp >> 1) * 32 < nrows;
  float ic[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t b = mx_scale_byte(fmaxf(cm[i], camax[warp ^ 1][8 * c + i]));
    ic[i] = mx_inv_scale(b);
    if ((warp & 1) == 0 && hrow == 0) scol_s[8 * c + i][warp >> 1] = blk_live ? (uint8_t)b : 0;
  }
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int row = r0 + rl0 + 2 * s + hrow;
    float f[8];
    unpack8(raw[s], f);
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = mx_encode2s(f[2 * i], f[2 * i + 1], ic[2 * i], ic[2 * i + 1]);
    if (row < nrows)
      *reinterpret_cast<uint2*>(codes_c + (size_t)row * cols + col) =
          make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
  }
  __syncthreads();   // the tile is read; the scale bytes are complete
  if (tid < 128) {
    const int mn = r0 + tid;
    if (mn < nrows)
      *reinterpret_cast<uint32_t*>(scales_r + mx_sf_offset(mn, c0 >> 5, cols / 128)) =
          *reinterpret_cast<const uint32_t*>(srow_s[tid]);
  } else if (tid < 256) {
    const int cc = tid - 128;
    *reinterpret_cast<uint32_t*>(scales_c + mx_sf_offset(c0 + cc, r0 >> 5, col_kchunks)) =
        *reinterpret_cast<const uint32_t*>(scol_s[cc]);
  }
  __syncthreads();   // camax and the scale staging are free again
}

// ------------------------------ both axes, TMA-fed persistent variant
// Persistent CTAs of 8 warps walk 128 x 128 tiles; each tile arrives in
// shared memory by TMA (two 64-column boxes, no swizzle) while the previous
// tile is quantised, so the bytes in flight do not depend on registers.
// Warp w takes rows 16w..16w+15 of the tile (half of one 32-row MX column
// block; warps 2b and 2b+1 combine their column maxima through shared
// memory), two rows per step with 16 lanes of 8 columns each (a 32-column
// row block is 4 lanes).  The first pass writes the row codes and keeps the
// raw rows in registers for the column codes of the second.
constexpr int kDualTile = 128;
constexpr int kDualTileBytes = kDualTile * kDualTile * 2;
constexpr int kDualWarps = 8;

#ifndef MOE_QDUAL_MIN_BLOCKS
#define MOE_QDUAL_MIN_BLOCKS 3     // resident CTAs per SM the register budget aims for
#endif
__global__ void __launch_bounds__(32 * kDualWarps, MOE_QDUAL_MIN_BLOCKS)
mx_quant_dual_tma_kernel(const __grid_constant__ CUtensorMap tin, int rows, int cols,
                         const int32_t* __restrict__ nrows_dev, uint8_t* __restrict__ codes_r,
                         uint8_t* __restrict__ scales_r, uint8_t* __restrict__ codes_c,
                         uint8_t* __restrict__ scales_c) {
  using namespace sm100;
  extern __shared__ __align__(128) uint8_t qsm[];
  __shared__ __align__(8) uint64_t full[2];
  __shared__ volatile int abort_flag;
  __shared__ __align__(16) float camax[kDualWarps][kDualTile];  // per-warp column maxima
  __shared__ __align__(4) uint8_t srow_s[kDualTile][4];          // row scale bytes, 4 K blocks
  __shared__ __align__(4) uint8_t scol_s[kDualTile][4];          // column scale bytes, 4 row blocks
  const int tid = threadIdx.x;
  const int nrows = nrows_dev ? min(*nrows_dev, rows) : rows;
  const int tiles_r = (nrows + kDualTile - 1) / kDualTile, tiles_c = cols / kDualTile;
  const int ntiles = tiles_r * tiles_c;
  if (tid == 0) {
    abort_flag = 0;
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    fence_barrier_init();
  }
  __syncthreads();
  auto issue = [&](int tile, int buf) {
    const int tr = tile / tiles_c, tc = tile % tiles_c;
    uint8_t* dst = qsm + buf * kDualTileBytes;
    mbar_arrive_expect_tx(&full[buf], kDualTileBytes);
    tma_load_2d(dst, &tin, &full[buf], tc * kDualTile, tr * kDualTile);
    tma_load_2d(dst + kDualTileBytes / 2, &tin, &full[buf], tc * kDualTile + 64, tr * kDualTile);
  };
  if (tid == 0 && (int)blockIdx.x < ntiles) issue(blockIdx.x, 0);
  uint32_t phase = 0;   // bit b: parity of full[b]
  int it = 0;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    const int buf = it & 1;
    if (tid == 0 && tile + (int)gridDim.x < ntiles) issue(tile + gridDim.x, buf ^ 1);
    if (!mbar_wait(&full[buf], (phase >> buf) & 1, &abort_flag, nullptr, 2000000000ull)) break;
    phase ^= 1u << buf;
    const int tr = tile / tiles_c, tc = tile % tiles_c;
    // TMA boxes: 64 columns x 128 rows each, rows of 128 bytes
    const uint8_t* t = qsm + buf * kDualTileBytes;
    auto chunk = [t](int rl, int c) {
      return t + (c >> 3) * (kDualTileBytes / 2) + rl * 128 + (c & 7) * 16;
    };
    mx_tile_both_axes(chunk, nullptr, tr * kDualTile, tc * kDualTile, nrows, cols, rows / 128,
                      codes_r, scales_r, codes_c, scales_c, camax, srow_s, scol_s);
  }
}

// -------------------------------------------- permute fused with MX codes
constexpr int kMaxK = 16;
constexpr int kWarps = 8;

__global__ void __launch_bounds__(32 * kWarps)
permute_mx_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ dst,
                  const int32_t* __restrict__ offsets, const int32_t* __restrict__ poff, int T,
                  int k, int d, int tok_blocks, uint4* __restrict__ Xp, uint8_t* __restrict__ Xq,
                  uint8_t* __restrict__ Xs) {
  const int d8 = d / 8;
  if ((int)blockIdx.x >= tok_blocks) {
    // pad rows of one group: bf16 zeros, zero codes, scale byte 0
    const int e = blockIdx.x - tok_blocks;
    const int r0 = poff[e] + (offsets[e + 1] - offsets[e]);
    const int r1 = poff[e + 1];
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (size_t i = threadIdx.x; i < (size_t)(r1 - r0) * d8; i += blockDim.x) {
      Xp[(size_t)r0 * d8 + i] = z;
      reinterpret_cast<uint2*>(Xq)[(size_t)r0 * d8 + i] = make_uint2(0, 0);
    }
    const int nkb = d / 32;
    for (int i = threadIdx.x; i < (r1 - r0) * nkb; i += blockDim.x)
      Xs[sf_offset(r0 + i / nkb, i % nkb, d / 128)] = 0;
    return;
  }
  const int t = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  int r[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) r[j] = j < k ? dst[(size_t)t * k + j] : -1;
  for (int seg = 0; seg * 256 < d; ++seg) {
    const int col = seg * 256 + lane * 8;
    const bool active = col < d;
    float f[8];
    float amax = 0.f;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (active) {
      v = ldg_stream(x + (size_t)t * d8 + col / 8);
      unpack8(v, f);
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    if (!active) continue;
    const uint32_t b = scale_byte(amax);
    const uint2 c = encode8(f, inv_scale(b));
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (r[j] < 0) continue;
      Xp[(size_t)r[j] * d8 + col / 8] = v;
      *reinterpret_cast<uint2*>(Xq + (size_t)r[j] * d + col) = c;
      if ((lane & 3) == 0) Xs[sf_offset(r[j], col / 32, d / 128)] = (uint8_t)b;
    }
  }
}


// ----------------------- dispatch straight into MX codes, both K axes
// Items of 128 rows x 128 columns of the expert-contiguous buffer (a
// 128-row tile never crosses a group: groups start on multiples of 128):
// row r is token src[r], or a zero row for src[r] < 0.  The item's rows are
// gathered into shared memory by coalesced 16-byte cp.async copies (two
// buffers: the next item loads while this one is quantised); each warp then
// quantises two of the item's sixteen 32 x 32 blocks (lane = row) along the
// rows (Xq / Xs, K = d: GEMM1) and down the columns (XqT / XsT, K = the
// padded rows: GEMM1 weight gradient), and the item's scale bytes leave as
// whole 32-bit words of the tensor-core layout.  The bf16 permuted copy is
// never written; rows from poff[E] on are not touched (no GEMM reads them).
//
// With a gate (the backward's dY rows): row r of group e is g * x[t] with
// g = gates[t, j] for the slot j of expert e in topk[t, :], rounded to bf16
// as the combine backward rounds it.
constexpr int kGatherWarps = 8;
constexpr int kGTile = 128;                     // rows and columns of an item
constexpr int kGRowBytes = kGTile * 2 + 16;     // padded shared-memory row (bank spread)
constexpr int kGBufBytes = kGTile * kGRowBytes;
constexpr int kGMaxE = 1024;                    // experts the gated mode accepts

struct GateRows {
  const float* gates;     // [T, k], null: no gate
  const int32_t* topk;    // [T, k]
  const int32_t* poff;    // [E + 1]
  int k, E;
};

using sm100::cp_async16;
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__global__ void __launch_bounds__(32 * kGatherWarps, 2)
permute_mx_gather_kernel(const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ src,
                         const int32_t* __restrict__ poff_end, int d, int A_pad_max,
                         uint8_t* __restrict__ Xq, uint8_t* __restrict__ Xs,
                         uint8_t* __restrict__ XqT, uint8_t* __restrict__ XsT, GateRows gr) {
  extern __shared__ __align__(16) uint8_t gsm[];          // 2 x kGBufBytes
  __shared__ int tok_s[2][kGTile];
  __shared__ float gate_s[2][kGTile];        // gates of the rows of the item in each buffer
  __shared__ int poff_s[kGMaxE + 1];         // group offsets (gated mode)
  __shared__ __align__(4) uint8_t srow_s[kGTile][4];      // row scale bytes, 4 K blocks
  __shared__ __align__(4) uint8_t scol_s[kGTile][4];      // column scale bytes, 4 row blocks
  __shared__ __align__(16) float camax[kGatherWarps][kGTile];  // per-warp column maxima
  const int nrows = min(*poff_end, A_pad_max);
  const int ctiles = d / kGTile;
  const int nitems = (nrows / kGTile) * ctiles;
  const int tid = threadIdx.x;

  // gather the item's rows into buffer `buf` (16 threads per 256-byte row)
  auto issue = [&](int item, int buf) {
    const int rt = item / ctiles, ct = item - rt * ctiles;
    const int r0 = rt * kGTile, c0 = ct * kGTile;
    uint8_t* dst = gsm + buf * kGBufBytes;
#pragma unroll
    for (int it = 0; it < kGTile * 16 / (32 * kGatherWarps); ++it) {
      const int i = tid + it * 32 * kGatherWarps;
      const int row = i >> 4, ch = i & 15;
      const int t = src[r0 + row];
      if (ch == 0) tok_s[buf][row] = t;
      const __nv_bfloat16* s = t >= 0 ? x + (size_t)t * d + c0 + ch * 8 : x;
      cp_async16(dst + row * kGRowBytes + ch * 16, s, t >= 0);
    }
    cp_async_commit();
  };

  // the gate of row `row` of the row tile at r0, whose token is t: the
  // tile's group is the largest e with poff[e] <= r0 (a non-empty one, as
  // r0 < poff[E]), the gate the token's slot of that expert
  auto group_of = [&](int r0) {
    int lo = 0, hi = gr.E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (poff_s[mid] <= r0) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  auto gate_of = [&](int e, int t) {
    float g = 0.f;
    if (t >= 0)
      for (int j = 0; j < gr.k; ++j)
        if (__ldg(gr.topk + (size_t)t * gr.k + j) == e) g = __ldg(gr.gates + (size_t)t * gr.k + j);
    return g;
  };
  if (gr.gates)
    for (int e = tid; e <= gr.E; e += blockDim.x) poff_s[e] = __ldg(gr.poff + e);

  int it = 0;
  if ((int)blockIdx.x < nitems) issue(blockIdx.x, 0);
  for (int item = blockIdx.x; item < nitems; item += gridDim.x, ++it) {
    const int buf = it & 1;
    const int nxt = item + gridDim.x;
    if (nxt < nitems) issue(nxt, buf ^ 1);
    else cp_async_commit();                    // keep the group count uniform
    cp_async_wait<1>();                        // this thread's copies of `item` landed
    __syncthreads();                           // everyone's have
    const int rt = item / ctiles, ct = item - rt * ctiles;
    const int r0 = rt * kGTile, c0 = ct * kGTile;
    // gated mode: the first item's gates now; every later item's are
    // prefetched (k <= 4: topk and gate words loaded here, used after the
    // quantisation below) and written to gate_s one item ahead
    int pe[4] = {-1, -1, -1, -1};
    float pg[4] = {0.f, 0.f, 0.f, 0.f};
    if (gr.gates) {
      if (it == 0) {
        if (tid < kGTile) gate_s[buf][tid] = gate_of(group_of(r0), tok_s[buf][tid]);
        __syncthreads();
      }
      if (tid < kGTile && nxt < nitems && gr.k <= 4) {
        const int tn = tok_s[buf ^ 1][tid];
        if (tn >= 0) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (j < gr.k) {
              pe[j] = __ldg(gr.topk + (size_t)tn * gr.k + j);
              pg[j] = __ldg(gr.gates + (size_t)tn * gr.k + j);
            }
          }
        }
      }
    }
    const uint8_t* tile = gsm + buf * kGBufBytes;
    auto chunk = [tile](int rl, int c) { return tile + rl * kGRowBytes + c * 16; };
    // gated rows: bf16(g * dout row), as the unfused dY holds it
    mx_tile_both_axes(chunk, gr.gates ? gate_s[buf] : nullptr, r0, c0, nrows, d, A_pad_max / 128,
                      Xq, Xs, XqT, XsT, camax, srow_s, scol_s);
    if (gr.gates && tid < kGTile && nxt < nitems) {
      // the next item's gates (read after the next item's first barrier)
      const int rn = (nxt / ctiles) * kGTile;
      const int e = group_of(rn);
      float gn = 0.f;
      if (gr.k <= 4) {
#pragma unroll
        for (int j = 0; j < 4; ++j) gn = pe[j] == e ? pg[j] : gn;
      } else {
        gn = gate_of(e, tok_s[buf ^ 1][tid]);
      }
      gate_s[buf ^ 1][tid] = gn;
    }
  }
  cp_async_wait<0>();
}

}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_permute_mx(const void* x, const int32_t* src, const int32_t* poff,
                                       int T, int d, int E, int A_pad_max, uint8_t* Xq,
                                       uint8_t* Xs, uint8_t* XqT, uint8_t* XsT,
                                       moe_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  MOE_CHECK_ARG(T > 0 && E > 0 && d > 0 && d % 128 == 0, "moe_permute_mx: d %% 128");
  MOE_CHECK_ARG(A_pad_max > 0 && A_pad_max % 128 == 0, "moe_permute_mx: A_pad_max %% 128");
  MOE_CHECK_ARG(x && src && poff && Xq && Xs && XqT && XsT, "moe_permute_mx: null pointer");
  MOE_CHECK_ARG(aligned16(x) && aligned16(Xq) && aligned16(XqT), "moe_permute_mx: unaligned buffer");
  const long long items = (long long)(A_pad_max / kGTile) * (d / kGTile);
  const int grid = (int)std::min<long long>(items, 2LL * num_sms());
  MOE_TRY(set_smem_limit(reinterpret_cast<const void*>(permute_mx_gather_kernel), 2 * kGBufBytes,
                         "moe_permute_mx"));
  permute_mx_gather_kernel<<<grid, 32 * kGatherWarps, 2 * kGBufBytes, s>>>(
      static_cast<const __nv_bfloat16*>(x), src, poff + E, d, A_pad_max, Xq, Xs, XqT, XsT,
      GateRows{nullptr, nullptr, nullptr, 0, E});
  MOE_CHECK_LAUNCH("moe_permute_mx");
  return MOE_OK;
}

extern "C" moe_status_t moe_combine_bwd_mx(const void* dout, const float* gates,
                                           const int32_t* topk_idx, const int32_t* src,
                                           const int32_t* poff, int T, int k, int d, int E,
                                           int A_pad_max, uint8_t* dYq, uint8_t* dYs,
                                           uint8_t* dYTq, uint8_t* dYTs, moe_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  MOE_CHECK_ARG(T > 0 && E > 0 && E <= kGMaxE && k > 0 && k <= 16 && d > 0 && d % 128 == 0,
                "moe_combine_bwd_mx: d %% 128, 0 < k <= 16, E <= 1024");
  MOE_CHECK_ARG(A_pad_max > 0 && A_pad_max % 128 == 0, "moe_combine_bwd_mx: A_pad_max %% 128");
  MOE_CHECK_ARG(dout && gates && topk_idx && src && poff && dYq && dYs && dYTq && dYTs,
                "moe_combine_bwd_mx: null pointer");
  MOE_CHECK_ARG(aligned16(dout) && aligned16(dYq) && aligned16(dYTq),
                "moe_combine_bwd_mx: unaligned buffer");
  const long long items = (long long)(A_pad_max / kGTile) * (d / kGTile);
  const int grid = (int)std::min<long long>(items, 2LL * num_sms());
  MOE_TRY(set_smem_limit(reinterpret_cast<const void*>(permute_mx_gather_kernel), 2 * kGBufBytes,
                         "moe_combine_bwd_mx"));
  permute_mx_gather_kernel<<<grid, 32 * kGatherWarps, 2 * kGBufBytes, s>>>(
      static_cast<const __nv_bfloat16*>(dout), src, poff + E, d, A_pad_max, dYq, dYs, dYTq, dYTs,
      GateRows{gates, topk_idx, poff, k, E});
  MOE_CHECK_LAUNCH("moe_combine_bwd_mx");
  return MOE_OK;
}

moe_status_t moe_permute_mx_launch(const void* x, const int32_t* dst, const int32_t* offsets,
                                   const int32_t* poff, int T, int k, int d, int E, int A_pad_max,
                                   void* Xp, uint8_t* Xq, uint8_t* Xs, cudaStream_t s) {
  MOE_CHECK_ARG(d % 128 == 0 && A_pad_max % 128 == 0, "moe_permute: MX needs d %% 128 == 0");
  MOE_CHECK_ARG(aligned16(Xq) && aligned16(Xs), "moe_permute: unaligned MX buffers");
  const int tok_blocks = (T + kWarps - 1) / kWarps;
  permute_mx_kernel<<<tok_blocks + E, 32 * kWarps, 0, s>>>(
      static_cast<const uint4*>(x), dst, offsets, poff, T, k, d, tok_blocks,
      static_cast<uint4*>(Xp), Xq, Xs);
  MOE_CHECK_LAUNCH("permute_mx");
  return MOE_OK;
}

extern "C" moe_status_t mx_quantize(const void* in, int rows, int cols, int axis,
                                    const int32_t* poff, int E, const int32_t* nrows_dev,
                                    uint8_t* codes, uint8_t* scales, moe_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  (void)poff;
  (void)E;
  MOE_CHECK_ARG(rows > 0 && cols > 0 && rows % 128 == 0 && cols % 128 == 0,
                "mx_quantize: rows and cols must be multiples of 128");
  MOE_CHECK_ARG(axis == 0 || axis == 1, "mx_quantize: axis must be 0 or 1");
  MOE_CHECK_ARG(in && codes && scales && aligned16(in) && aligned16(codes),
                "mx_quantize: null or unaligned pointer");
  const int segs = (cols + 255) / 256;
  const int warps_per_block = 8;
  if (axis == 0) {
    const long long warps = (long long)rows * segs;
    const long long blocks = (warps + warps_per_block - 1) / warps_per_block;
    mx_quant_rows_kernel<<<(unsigned)blocks, 32 * warps_per_block, 0, s>>>(
        static_cast<const uint4*>(in), rows, cols, nrows_dev, codes, scales);
  } else {
    const long long warps = (long long)(rows / 32) * segs;
    const long long blocks = (warps + warps_per_block - 1) / warps_per_block;
    mx_quant_cols_kernel<<<(unsigned)blocks, 32 * warps_per_block, 0, s>>>(
        static_cast<const __nv_bfloat16*>(in), rows, cols, nrows_dev, codes, scales);
  }
  MOE_CHECK_LAUNCH("mx_quantize");
  return MOE_OK;
}

extern "C" moe_status_t mx_quantize_dual(const void* in, int rows, int cols,
                                         const int32_t* nrows_dev, uint8_t* codes_rows,
                                         uint8_t* scales_rows, uint8_t* codes_cols,
                                         uint8_t* scales_cols, moe_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  MOE_CHECK_ARG(rows > 0 && cols > 0 && rows % 128 == 0 && cols % 128 == 0,
                "mx_quantize_dual: rows and cols must be multiples of 128");
  MOE_CHECK_ARG(in && codes_rows && scales_rows && codes_cols && scales_cols && aligned16(in) &&
                    aligned16(codes_rows) && aligned16(codes_cols),
                "mx_quantize_dual: null or unaligned pointer");
  auto fn = tensor_map_encoder();
  if (!fn) {
    set_error("mx_quantize_dual: cuTensorMapEncodeTiled unavailable");
    return MOE_ERR_CUDA;
  }
  CUtensorMap m;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  if (fn(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(in), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
    set_error("mx_quantize_dual: tensor map encoding failed");
    return MOE_ERR_CUDA;
  }
  const size_t smem = 2 * (size_t)kDualTileBytes;
  MOE_TRY(set_smem_limit(reinterpret_cast<const void*>(mx_quant_dual_tma_kernel), smem,
                         "mx_quantize_dual"));
  const long long ntiles = (long long)(rows / 128) * (cols / 128);
  const int grid = (int)std::min<long long>(ntiles, (long long)MOE_QDUAL_MIN_BLOCKS * num_sms());
  mx_quant_dual_tma_kernel<<<grid, 32 * kDualWarps, smem, s>>>(m, rows, cols, nrows_dev, codes_rows,
                                                   scales_rows, codes_cols, scales_cols);
  MOE_CHECK_LAUNCH("mx_quantize_dual");
  return MOE_OK;
}
