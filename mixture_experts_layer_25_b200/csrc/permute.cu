// Rowwise dispatch into expert-contiguous buffers, the gate-weighted
// combine, and their backward passes (HBM-bound gathers/scatters).
//
// Olmo-core 3 オープン混合エキスパート学習インフラストラクチャ, section
// "ルーティングと計算の最適化": routed tokens are written straight into the
// experts' input buffers.  Every kernel moves whole token rows with 16-byte
// vector accesses, each row read once.
#include <type_traits>

#include <algorithm>

#include "common.cuh"

namespace moe {

constexpr int kTopKLimit = 16;

// call f(std::integral_constant<int, KM>) with the smallest KM in
// {2, 4, 8, 16} >= k: the kernels keep k rows' state in register arrays
template <class F>
void dispatch_k(int k, F&& f) {
  if (k <= 2) f(std::integral_constant<int, 2>{});
  else if (k <= 4) f(std::integral_constant<int, 4>{});
  else if (k <= 8) f(std::integral_constant<int, 8>{});
  else f(std::integral_constant<int, 16>{});
}

// zero the pad rows [poff[e] + counts[e], poff[e+1]) of one expert group
// (and, when given, the same entries of a per-row fp32 vector)
__device__ __forceinline__ void zero_pad_rows(const int32_t* offsets, const int32_t* poff, int e,
                                              int d8, uint4* buf, float* row_vec = nullptr) {
  const int r0 = poff[e] + (offsets[e + 1] - offsets[e]);
  const int r1 = poff[e + 1];
  const size_t n = (size_t)(r1 - r0) * d8;
  const uint4 z = make_uint4(0, 0, 0, 0);
  if (buf) {
    uint4* base = buf + (size_t)r0 * d8;
    for (size_t i = threadIdx.x; i < n; i += blockDim.x) base[i] = z;
  }
  if (row_vec)
    for (int r = r0 + (int)threadIdx.x; r < r1; r += blockDim.x) row_vec[r] = 0.f;
}

// Row teams: `tpt` threads (a multiple of 32, at most 256) share one token
// row, each moving 16-byte chunks lt, lt + tpt, ...; a 256-thread block holds
// 256 / tpt tokens.  With d = 2048 a whole block works on one row, so every
// load of the row is in flight at once.
constexpr int kBlock = 256;
// The gather-reduce kernels keep all k row loads of a chunk in flight at
// once; their occupancy is set by registers.  unpermute_sum (which also
// gathers fp32 router-weight rows) is held to 64 registers so that four
// blocks stay resident per SM (measured 1.35x faster at d = 2048, 3x at
// d = 6144, k = 8); combine_bwd runs its single chunk per thread without
// unrolling (64 registers at k = 4).
constexpr int kUnpermuteMinBlocks = 4;

__host__ __device__ __forceinline__ int team_threads(int d8) {
  return d8 >= kBlock ? kBlock : ((d8 + 31) / 32) * 32;
}

// ------------------------------------------------------------------ permute
template <int kMaxK>
__global__ void __launch_bounds__(kBlock)
permute_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ dst,
               const int32_t* __restrict__ offsets, const int32_t* __restrict__ poff, int T,
               int k, int d8, int tok_blocks, uint4* __restrict__ Xp) {
  if ((int)blockIdx.x >= tok_blocks) {
    zero_pad_rows(offsets, poff, blockIdx.x - tok_blocks, d8, Xp);
    return;
  }
  const int tpt = team_threads(d8);
  const int t = blockIdx.x * (kBlock / tpt) + threadIdx.x / tpt;
  const int lt = threadIdx.x % tpt;
  if (t >= T) return;
  int r[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) r[j] = j < k ? dst[(size_t)t * k + j] : -1;
  const uint4* xr = x + (size_t)t * d8;
#pragma unroll 2
  for (int c = lt; c < d8; c += tpt) {
    const uint4 v = ldg_stream(xr + c);
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (r[j] >= 0) Xp[(size_t)r[j] * d8 + c] = v;
  }
}

// Persistent form for rows of at most kBlock 16-byte chunks and k <= 4: the
// next token's row and routing entries are loaded while the current row is
// written to its k slots.  Blocks from nblocks on zero the pad rows.
template <int kMaxK>
__global__ void __launch_bounds__(kBlock, 3)
permute_pf_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ dst,
                  const int32_t* __restrict__ offsets, const int32_t* __restrict__ poff, int T,
                  int k, int d8, int nblocks, uint4* __restrict__ Xp) {
  if ((int)blockIdx.x >= nblocks) {
    zero_pad_rows(offsets, poff, blockIdx.x - nblocks, d8, Xp);
    return;
  }
  const int tpt = team_threads(d8);
  const int tpb = kBlock / tpt;
  const int team = threadIdx.x / tpt, lt = threadIdx.x % tpt;
  if (lt >= d8) return;                      // no block-wide barriers below
  const int stride = nblocks * tpb;
  auto load_meta = [&](int t, int* r) {
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) r[j] = (t < T && j < k) ? dst[(size_t)t * k + j] : -1;
  };
  int t = blockIdx.x * tpb + team;
  int r[kMaxK];
  uint4 v = make_uint4(0, 0, 0, 0);
  load_meta(t, r);
  if (t < T) v = ldg_stream(x + (size_t)t * d8 + lt);
  for (; t < T; t += stride) {
    const int tn = t + stride;
    int rn[kMaxK];
    load_meta(tn, rn);
    uint4 vn = make_uint4(0, 0, 0, 0);
    if (tn < T) vn = ldg_stream(x + (size_t)tn * d8 + lt);
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (r[j] >= 0) Xp[(size_t)r[j] * d8 + lt] = v;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) r[j] = rn[j];
    v = vn;
  }
}

// ------------------------------------------------------------------ combine
template <int kMaxK>
__global__ void __launch_bounds__(kBlock)
combine_kernel(const uint4* __restrict__ Y, const float* __restrict__ gates,
               const int32_t* __restrict__ dst, int T, int k, int d8, uint4* __restrict__ out) {
  const int tpt = team_threads(d8);
  const int t = blockIdx.x * (kBlock / tpt) + threadIdx.x / tpt;
  const int lt = threadIdx.x % tpt;
  if (t >= T) return;
  int r[kMaxK];
  float g[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    r[j] = j < k ? dst[(size_t)t * k + j] : -1;
    g[j] = (j < k && gates) ? gates[(size_t)t * k + j] : 1.f;
  }
#pragma unroll 2
  for (int c = lt; c < d8; c += tpt) {
    uint4 v[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (r[j] >= 0) v[j] = ldg_stream(Y + (size_t)r[j] * d8 + c);
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (r[j] < 0) continue;
      float f[8];
      unpack8(v[j], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(g[j], f[i], acc[i]);
    }
    out[(size_t)t * d8 + c] = pack8(acc);
  }
}

// Persistent form of the k-row gather-sum (combine with gates, the dx sum
// without) for rows of at most kBlock 16-byte chunks and k <= 4: each team
// walks tokens with a stride of the whole grid, and the next token's k rows
// (and the routing entries of the one after) are loaded while the current
// token is summed.  Same per-element arithmetic as combine_kernel /
// unpermute_sum_kernel.
template <int kMaxK, bool kGated>
__global__ void __launch_bounds__(kBlock, 3)
gather_sum_pf_kernel(const uint4* __restrict__ rows, const float* __restrict__ gates,
                     const int32_t* __restrict__ dst, int T, int k, int d8, int nblocks,
                     uint4* __restrict__ out) {
  const int tpt = team_threads(d8);
  const int tpb = kBlock / tpt;
  const int team = threadIdx.x / tpt, lt = threadIdx.x % tpt;
  if (lt >= d8) return;                      // no block-wide barriers below
  const int stride = nblocks * tpb;
  auto load_meta = [&](int t, int* r, float* g) {
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      const bool on = t < T && j < k;
      r[j] = on ? dst[(size_t)t * k + j] : -1;
      g[j] = (on && kGated) ? gates[(size_t)t * k + j] : 1.f;
    }
  };
  auto load_rows = [&](const int* r, uint4* v) {
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (r[j] >= 0) v[j] = ldg_stream(rows + (size_t)r[j] * d8 + lt);
  };
  int t = blockIdx.x * tpb + team;
  int r[kMaxK], rn[kMaxK];
  float g[kMaxK], gn[kMaxK];
  uint4 v[kMaxK];
  load_meta(t, r, g);
  load_rows(r, v);
  load_meta(t + stride, rn, gn);
  for (; t < T; t += stride) {
    uint4 vn[kMaxK];
    load_rows(rn, vn);
    int rn2[kMaxK];
    float gn2[kMaxK];
    load_meta(t + 2 * stride, rn2, gn2);
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (r[j] < 0) continue;
      float f[8];
      unpack8(v[j], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = kGated ? fmaf(g[j], f[i], acc[i]) : acc[i] + f[i];
    }
    out[(size_t)t * d8 + lt] = pack8(acc);
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      r[j] = rn[j]; g[j] = gn[j]; v[j] = vn[j];
      rn[j] = rn2[j]; gn[j] = gn2[j];
    }
  }
}

// launch the persistent gather-sum if it applies (d <= 2048, k <= 4)
template <bool kGated>
bool launch_gather_sum_pf(const void* rows, const float* gates, const int32_t* dst, int T, int k,
                          int d8, void* out, cudaStream_t s) {
  if (d8 > kBlock || k > 4) return false;
  const int tpb = kBlock / team_threads(d8);
  const int nblocks = std::min((T + tpb - 1) / tpb, 3 * num_sms());
  auto go = [&](auto KM) {
    gather_sum_pf_kernel<decltype(KM)::value, kGated><<<nblocks, kBlock, 0, s>>>(
        static_cast<const uint4*>(rows), gates, dst, T, k, d8, nblocks, static_cast<uint4*>(out));
  };
  if (k <= 2) go(std::integral_constant<int, 2>{});
  else go(std::integral_constant<int, 4>{});
  return true;
}

// ------------------------------------------------------- combine backward
template <int kMaxK>
__global__ void __launch_bounds__(kBlock)
combine_bwd_kernel(const uint4* __restrict__ dout, const uint4* __restrict__ Y,
                   const float* __restrict__ gates, const int32_t* __restrict__ dst,
                   const int32_t* __restrict__ offsets, const int32_t* __restrict__ poff, int T,
                   int k, int d8, int tok_blocks, uint4* __restrict__ dY, float* __restrict__ dg,
                   float* __restrict__ dl, float* __restrict__ dl_rows) {
  if ((int)blockIdx.x >= tok_blocks) {
    zero_pad_rows(offsets, poff, blockIdx.x - tok_blocks, d8, dY, dl_rows);
    return;
  }
  __shared__ float red[kBlock / 32][kMaxK];
  const int tpt = team_threads(d8);
  const int t = blockIdx.x * (kBlock / tpt) + threadIdx.x / tpt;
  const int lt = threadIdx.x % tpt;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool live = t < T;
  int r[kMaxK];
  float g[kMaxK], dot[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    r[j] = (live && j < k) ? dst[(size_t)t * k + j] : -1;
    g[j] = (live && j < k) ? gates[(size_t)t * k + j] : 0.f;
    dot[j] = 0.f;
  }
  if (live) {
#pragma unroll 1
    for (int c = lt; c < d8; c += tpt) {
      const uint4 dv = ldg_stream(dout + (size_t)t * d8 + c);
      uint4 yv[kMaxK];
#pragma unroll
      for (int j = 0; j < kMaxK; ++j)
        if (r[j] >= 0) yv[j] = ldg_stream(Y + (size_t)r[j] * d8 + c);
      float fd[8];
      unpack8(dv, fd);
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        if (r[j] < 0) continue;
        float fy[8], sc[8];
        unpack8(yv[j], fy);
        float sdot = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          sdot = fmaf(fd[i], fy[i], sdot);
          sc[i] = g[j] * fd[i];
        }
        dot[j] += sdot;
        if (dY) dY[(size_t)r[j] * d8 + c] = pack8(sc);
      }
    }
  }
  // team reduction of the k dot products: warps, then the team's warps
#pragma unroll
  for (int j = 0; j < kMaxK; ++j)
    if (j < k) dot[j] = warp_sum(dot[j]);
  if (lane == 0)
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (j < k) red[warp][j] = dot[j];
  __syncthreads();
  if (!live || lt != 0) return;
  const int w0 = warp, nw = tpt / 32;
  float gs = 0.f;
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    if (j >= k) continue;
    float s = 0.f;
    for (int w = 0; w < nw; ++w) s += red[w0 + w][j];
    dot[j] = s;
    gs = fmaf(g[j], s, gs);
  }
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    if (j >= k) continue;
    dg[(size_t)t * k + j] = dot[j];
    if (dl) {
      const float v = g[j] * (dot[j] - gs);
      dl[(size_t)t * k + j] = v;
      if (dl_rows && r[j] >= 0) dl_rows[r[j]] = v;
    }
  }
}

// Persistent form for rows of at most kBlock 16-byte chunks (d <= 2048):
// one chunk per thread, and while a token is reduced the loads of the next
// token's rows (and the routing entries of the one after) are already in
// flight, so the bytes in flight do not drop between tokens.  Same results
// as combine_bwd_kernel (same per-thread arithmetic and reduction order).
template <int kMaxK>
__global__ void __launch_bounds__(kBlock, 3)
combine_bwd_pf_kernel(const uint4* __restrict__ dout, const uint4* __restrict__ Y,
                      const float* __restrict__ gates, const int32_t* __restrict__ dst,
                      const int32_t* __restrict__ offsets, const int32_t* __restrict__ poff, int T,
                      int k, int d8, int tok_blocks, uint4* __restrict__ dY, float* __restrict__ dg,
                      float* __restrict__ dl, float* __restrict__ dl_rows) {
  if ((int)blockIdx.x >= tok_blocks) {
    zero_pad_rows(offsets, poff, blockIdx.x - tok_blocks, d8, dY, dl_rows);
    return;
  }
  __shared__ float red[kBlock / 32][kMaxK];
  const int tpt = team_threads(d8);
  const int tpb = kBlock / tpt;
  const int team = threadIdx.x / tpt, lt = threadIdx.x % tpt;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int stride = tok_blocks * tpb;
  const bool has_c = lt < d8;
  auto load_meta = [&](int t, int* r, float* g) {
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      const bool on = t < T && j < k;
      r[j] = on ? dst[(size_t)t * k + j] : -1;
      g[j] = on ? gates[(size_t)t * k + j] : 0.f;
    }
  };
  auto load_rows = [&](int t, const int* r, uint4& dv, uint4* yv) {
    if (t < T && has_c) {
      dv = ldg_stream(dout + (size_t)t * d8 + lt);
#pragma unroll
      for (int j = 0; j < kMaxK; ++j)
        if (r[j] >= 0) yv[j] = ldg_stream(Y + (size_t)r[j] * d8 + lt);
    }
  };
  int base = blockIdx.x * tpb;
  int r[kMaxK], rn[kMaxK];
  float g[kMaxK], gn[kMaxK];
  uint4 dv = make_uint4(0, 0, 0, 0), yv[kMaxK];
  load_meta(base + team, r, g);
  load_rows(base + team, r, dv, yv);
  load_meta(base + stride + team, rn, gn);
  for (; base < T; base += stride) {            // block-uniform trip count
    const int t = base + team;
    const bool live = t < T;
    // next token: its rows now, the routing entries of the one after
    uint4 dvn = make_uint4(0, 0, 0, 0), yvn[kMaxK];
    load_rows(t + stride, rn, dvn, yvn);
    int rn2[kMaxK];
    float gn2[kMaxK];
    load_meta(t + 2 * stride, rn2, gn2);

    float dot[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) dot[j] = 0.f;
    if (live && has_c) {
      float fd[8];
      unpack8(dv, fd);
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        if (r[j] < 0) continue;
        float fy[8], sc[8];
        unpack8(yv[j], fy);
        float sdot = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          sdot = fmaf(fd[i], fy[i], sdot);
          sc[i] = g[j] * fd[i];
        }
        dot[j] += sdot;
        if (dY) dY[(size_t)r[j] * d8 + lt] = pack8(sc);
      }
    }
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (j < k) dot[j] = warp_sum(dot[j]);
    if (lane == 0)
#pragma unroll
      for (int j = 0; j < kMaxK; ++j)
        if (j < k) red[warp][j] = dot[j];
    __syncthreads();
    if (live && lt == 0) {
      const int w0 = warp, nw = tpt / 32;
      float gs = 0.f;
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        if (j >= k) continue;
        float sum = 0.f;
        for (int w = 0; w < nw; ++w) sum += red[w0 + w][j];
        dot[j] = sum;
        gs = fmaf(g[j], sum, gs);
      }
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        if (j >= k) continue;
        dg[(size_t)t * k + j] = dot[j];
        if (dl) {
          const float v = g[j] * (dot[j] - gs);
          dl[(size_t)t * k + j] = v;
          if (dl_rows && r[j] >= 0) dl_rows[r[j]] = v;
        }
      }
    }
    __syncthreads();                            // red is reused by the next token
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      r[j] = rn[j]; g[j] = gn[j]; yv[j] = yvn[j];
      rn[j] = rn2[j]; gn[j] = gn2[j];
    }
    dv = dvn;
  }
}

// ------------------------------------------------- dispatch backward (dx)
__global__ void transpose_f32_kernel(const float* __restrict__ in, int rows, int cols,
                                     float* __restrict__ out) {
  __shared__ float tile[32][33];
  const int bx = blockIdx.x * 32, by = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = by + i, c = bx + threadIdx.x;
    if (r < rows && c < cols) tile[i][threadIdx.x] = in[(size_t)r * cols + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = bx + i, c = by + threadIdx.x;   // out is [cols, rows]
    if (r < cols && c < rows) out[(size_t)r * rows + c] = tile[threadIdx.x][i];
  }
}

template <int kMaxK>
__global__ void __launch_bounds__(kBlock, kUnpermuteMinBlocks)
unpermute_sum_kernel(const uint4* __restrict__ dXp, const int32_t* __restrict__ dst,
                     const int32_t* __restrict__ topk_idx, const float* __restrict__ dl,
                     const float* __restrict__ WrT /* [E,d] or null */, int T, int k, int d8,
                     int E, uint4* __restrict__ dx) {
  const int tpt = team_threads(d8);
  const int t = blockIdx.x * (kBlock / tpt) + threadIdx.x / tpt;
  const int lt = threadIdx.x % tpt;
  if (t >= T) return;
  int r[kMaxK], e[kMaxK];
  float w[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    r[j] = j < k ? dst[(size_t)t * k + j] : -1;
    e[j] = (j < k && WrT) ? topk_idx[(size_t)t * k + j] : -1;
    w[j] = (j < k && WrT) ? dl[(size_t)t * k + j] : 0.f;
    if (e[j] >= E) e[j] = -1;
  }
#pragma unroll 1
  for (int c = lt; c < d8; c += tpt) {
    uint4 v[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (r[j] >= 0) v[j] = ldg_stream(dXp + (size_t)r[j] * d8 + c);
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (r[j] < 0) continue;
      float f[8];
      unpack8(v[j], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += f[i];
    }
    if (WrT) {
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        if (r[j] < 0 || e[j] < 0) continue;
        const float4* wr = reinterpret_cast<const float4*>(WrT + (size_t)e[j] * d8 * 8) + 2 * c;
        const float4 a = __ldg(wr), b = __ldg(wr + 1);
        acc[0] = fmaf(w[j], a.x, acc[0]); acc[1] = fmaf(w[j], a.y, acc[1]);
        acc[2] = fmaf(w[j], a.z, acc[2]); acc[3] = fmaf(w[j], a.w, acc[3]);
        acc[4] = fmaf(w[j], b.x, acc[4]); acc[5] = fmaf(w[j], b.y, acc[5]);
        acc[6] = fmaf(w[j], b.z, acc[6]); acc[7] = fmaf(w[j], b.w, acc[7]);
      }
    }
    dx[(size_t)t * d8 + c] = pack8(acc);
  }
}

// --------------------------------------------------------- router wgrad
// dWr[i, e] = sum over the real rows r of group e of x[src[r], i] * dl_rows[r].
// Pass 1: every 128-row block of the permuted buffer (one expert's rows, as
// groups start on multiples of 128) sums its rows into P[block][:]; pass 2
// adds the blocks of each expert.  Work spreads evenly however skewed the
// load, and the summation order is fixed.
constexpr int kRwRowGroups = 8;
__global__ void __launch_bounds__(256)
router_wgrad_blocks_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ src,
                           const float* __restrict__ dl_rows, const int32_t* __restrict__ poff,
                           int E, int d8, float* __restrict__ P) {
  __shared__ float red[kRwRowGroups][256 + 4];
  const int blk = blockIdx.x;
  if (blk * 128 >= poff[E]) return;
  const int rg = threadIdx.x >> 5, cl = threadIdx.x & 31;
  const int c = blockIdx.y * 32 + cl;       // 8-column chunk index
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (c < d8) {
#pragma unroll 4
    for (int i = rg; i < 128; i += kRwRowGroups) {
      const int r = blk * 128 + i;
      const int t = src[r];
      if (t < 0) continue;                  // pad row
      const float w = dl_rows[r];
      float f[8];
      unpack8(x[(size_t)t * d8 + c], f);
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] = fmaf(f[q], w, acc[q]);
    }
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) red[rg][cl * 8 + q] = acc[q];
  __syncthreads();
  const int col = blockIdx.y * 256 + threadIdx.x;
  if (col < d8 * 8) {
    float sum = 0.f;
#pragma unroll
    for (int g = 0; g < kRwRowGroups; ++g) sum += red[g][threadIdx.x];
    P[(size_t)blk * d8 * 8 + col] = sum;
  }
}

__global__ void __launch_bounds__(256)
router_wgrad_reduce_kernel(const float* __restrict__ P, const int32_t* __restrict__ poff, int E,
                           int d, float* __restrict__ dWr) {
  const int e = blockIdx.x;
  const int col = blockIdx.y * 256 + threadIdx.x;
  if (col >= d) return;
  float sum = 0.f;
  for (int b = poff[e] / 128; b < poff[e + 1] / 128; ++b) sum += P[(size_t)b * d + col];
  dWr[(size_t)col * E + e] = sum;
}

}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_permute(const void* x, const int32_t* dst, const int32_t* offsets,
                                    const int32_t* poff, int T, int k, int d, int E,
                                    int A_pad_max, void* Xp, uint8_t* Xq, uint8_t* Xs,
                                    moe_stream_t stream);

moe_status_t moe_permute_mx_launch(const void* x, const int32_t* dst, const int32_t* offsets,
                                   const int32_t* poff, int T, int k, int d, int E, int A_pad_max,
                                   void* Xp, uint8_t* Xq, uint8_t* Xs, cudaStream_t s);

extern "C" moe_status_t moe_permute(const void* x, const int32_t* dst, const int32_t* offsets,
                                    const int32_t* poff, int T, int k, int d, int E,
                                    int A_pad_max, void* Xp, uint8_t* Xq, uint8_t* Xs,
                                    moe_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  MOE_CHECK_ARG(T > 0 && k > 0 && k <= kTopKLimit && E > 0 && d > 0 && d % 8 == 0,
                "moe_permute: bad T/k/E/d");
  MOE_CHECK_ARG(x && dst && offsets && poff && Xp && aligned16(x) && aligned16(Xp),
                "moe_permute: null or unaligned pointer");
  MOE_CHECK_ARG((Xq == nullptr) == (Xs == nullptr), "moe_permute: Xq and Xs go together");
  (void)A_pad_max;
  if (Xq) return moe_permute_mx_launch(x, dst, offsets, poff, T, k, d, E, A_pad_max, Xp, Xq, Xs, s);
  const int tpb = kBlock / team_threads(d / 8);
  const int tok_blocks = (T + tpb - 1) / tpb;
  if (d / 8 <= kBlock && k <= 4) {
    const int nblocks = std::min(tok_blocks, 3 * num_sms());
    auto go = [&](auto KM) {
      permute_pf_kernel<decltype(KM)::value><<<nblocks + E, kBlock, 0, s>>>(
          static_cast<const uint4*>(x), dst, offsets, poff, T, k, d / 8, nblocks,
          static_cast<uint4*>(Xp));
    };
    if (k <= 2) go(std::integral_constant<int, 2>{});
    else go(std::integral_constant<int, 4>{});
    MOE_CHECK_LAUNCH("permute");
    return MOE_OK;
  }
  dispatch_k(k, [&](auto KM) {
    permute_kernel<decltype(KM)::value><<<tok_blocks + E, kBlock, 0, s>>>(static_cast<const uint4*>(x), dst, offsets, poff, T, k, d / 8, tok_blocks,
      static_cast<uint4*>(Xp));
  });
  MOE_CHECK_LAUNCH("permute");
  return MOE_OK;
}

extern "C" moe_status_t moe_unpermute_combine(const void* Y, const float* gates,
                                              const int32_t* dst, int T, int k, int d, void* out,
                                              moe_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  MOE_CHECK_ARG(T > 0 && k > 0 && k <= kTopKLimit && d > 0 && d % 8 == 0, "moe_unpermute_combine: bad sizes");
  MOE_CHECK_ARG(Y && dst && out && aligned16(Y) && aligned16(out),
                "moe_unpermute_combine: null or unaligned pointer");
  const int tpb = kBlock / team_threads(d / 8);
  const int blocks = (T + tpb - 1) / tpb;
  const bool pf = gates ? launch_gather_sum_pf<true>(Y, gates, dst, T, k, d / 8, out, s)
                        : launch_gather_sum_pf<false>(Y, nullptr, dst, T, k, d / 8, out, s);
  if (!pf)
    dispatch_k(k, [&](auto KM) {
      combine_kernel<decltype(KM)::value><<<blocks, kBlock, 0, s>>>(static_cast<const uint4*>(Y), gates, dst,
                                                          T, k, d / 8, static_cast<uint4*>(out));
    });
  MOE_CHECK_LAUNCH("combine");
  return MOE_OK;
}

extern "C" moe_status_t moe_combine_bwd(const void* dout, const void* Y, const float* gates,
                                        const int32_t* dst, const int32_t* offsets,
                                        const int32_t* poff, int T, int k, int d, int E, void* dY,
                                        float* dg, float* dl, float* dl_rows,
                                        moe_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  MOE_CHECK_ARG(T > 0 && k > 0 && k <= kTopKLimit && E > 0 && d > 0 && d % 8 == 0,
                "moe_combine_bwd: bad sizes");
  MOE_CHECK_ARG(dout && Y && gates && dst && offsets && poff && dg,
                "moe_combine_bwd: null pointer");
  MOE_CHECK_ARG(aligned16(dout) && aligned16(Y) && (!dY || aligned16(dY)),
                "moe_combine_bwd: unaligned");
  const int tpb = kBlock / team_threads(d / 8);
  const int tok_blocks = (T + tpb - 1) / tpb;
  if (d / 8 <= kBlock && k <= 4) {
    // persistent: three resident blocks per SM walk the tokens (80 registers
    // at k <= 4; larger k would spill with two tokens' rows in registers)
    const int pblocks = std::min(tok_blocks, 3 * num_sms());
    auto go = [&](auto KM) {
      combine_bwd_pf_kernel<decltype(KM)::value><<<pblocks + E, kBlock, 0, s>>>(
          static_cast<const uint4*>(dout), static_cast<const uint4*>(Y), gates, dst, offsets, poff,
          T, k, d / 8, pblocks, static_cast<uint4*>(dY), dg, dl, dl_rows);
    };
    if (k <= 2) go(std::integral_constant<int, 2>{});
    else go(std::integral_constant<int, 4>{});
  } else {
    dispatch_k(k, [&](auto KM) {
      combine_bwd_kernel<decltype(KM)::value><<<tok_blocks + E, kBlock, 0, s>>>(static_cast<const uint4*>(dout), static_cast<const uint4*>(Y), gates, dst, offsets, poff, T,
        k, d / 8, tok_blocks, static_cast<uint4*>(dY), dg, dl, dl_rows);
    });
  }
  MOE_CHECK_LAUNCH("combine_bwd");
  return MOE_OK;
}

extern "C" size_t moe_unpermute_sum_workspace_size(int d, int E) {
  if (d <= 0 || E <= 0) return 0;
  return round_up((size_t)d * E * sizeof(float), 256);
}

extern "C" moe_status_t moe_unpermute_sum(const void* dXp, const int32_t* dst,
                                          const int32_t* topk_idx, const float* dl,
                                          const float* Wr, int T, int k, int d, int E, void* dx,
                                          void* ws, size_t ws_bytes, moe_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  MOE_CHECK_ARG(T > 0 && k > 0 && k <= kTopKLimit && d > 0 && d % 8 == 0 && E > 0,
                "moe_unpermute_sum: bad sizes");
  MOE_CHECK_ARG(dXp && dst && dx && aligned16(dXp) && aligned16(dx),
                "moe_unpermute_sum: null or unaligned pointer");
  float* WrT = nullptr;
  if (Wr) {
    MOE_CHECK_ARG(topk_idx && dl, "moe_unpermute_sum: router term needs topk_idx and dl");
    const size_t need = moe_unpermute_sum_workspace_size(d, E);
    if (!ws || ws_bytes < need) {
      set_error("moe_unpermute_sum: workspace %zu < %zu bytes", ws_bytes, need);
      return MOE_ERR_WORKSPACE;
    }
    MOE_CHECK_ARG(aligned16(ws), "moe_unpermute_sum: unaligned workspace");
    WrT = static_cast<float*>(ws);
    MOE_TRY(transpose_f32(Wr, d, E, WrT, s));
  }
  const int tpb = kBlock / team_threads(d / 8);
  const int blocks = (T + tpb - 1) / tpb;
  if (WrT || !launch_gather_sum_pf<false>(dXp, nullptr, dst, T, k, d / 8, dx, s))
    dispatch_k(k, [&](auto KM) {
      unpermute_sum_kernel<decltype(KM)::value><<<blocks, kBlock, 0, s>>>(static_cast<const uint4*>(dXp), dst, topk_idx, dl, WrT, T, k, d / 8, E,
        static_cast<uint4*>(dx));
    });
  MOE_CHECK_LAUNCH("unpermute_sum");
  return MOE_OK;
}

moe_status_t moe::transpose_f32(const float* in, int rows, int cols, float* out,
                                cudaStream_t s) {
  dim3 grid((cols + 31) / 32, (rows + 31) / 32), block(32, 8);
  transpose_f32_kernel<<<grid, block, 0, s>>>(in, rows, cols, out);
  MOE_CHECK_LAUNCH("transpose_f32");
  return MOE_OK;
}

extern "C" size_t moe_router_wgrad_workspace_size(int d, int A_pad_max) {
  if (d <= 0 || A_pad_max <= 0) return 0;
  return round_up((size_t)((A_pad_max + 127) / 128) * d * sizeof(float), 256);
}

extern "C" moe_status_t moe_router_wgrad(const void* x, const int32_t* src, const float* dl_rows,
                                         const int32_t* offsets, const int32_t* poff, int T,
                                         int d, int E, int A_pad_max, float* dWr, void* ws,
                                         size_t ws_bytes, moe_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  (void)offsets;
  MOE_CHECK_ARG(T > 0 && d > 0 && d % 8 == 0 && E > 0 && A_pad_max > 0,
                "moe_router_wgrad: bad sizes");
  MOE_CHECK_ARG(x && src && dl_rows && poff && dWr && aligned16(x),
                "moe_router_wgrad: null or unaligned pointer");
  const size_t need = moe_router_wgrad_workspace_size(d, A_pad_max);
  if (!ws || ws_bytes < need) {
    set_error("moe_router_wgrad: workspace %zu < %zu bytes", ws_bytes, need);
    return MOE_ERR_WORKSPACE;
  }
  float* P = static_cast<float*>(ws);
  dim3 g1((A_pad_max + 127) / 128, (d + 255) / 256);
  router_wgrad_blocks_kernel<<<g1, 256, 0, s>>>(static_cast<const uint4*>(x), src, dl_rows, poff,
                                                E, d / 8, P);
  MOE_CHECK_LAUNCH("router_wgrad_blocks");
  dim3 g2(E, (d + 255) / 256);
  router_wgrad_reduce_kernel<<<g2, 256, 0, s>>>(P, poff, E, d, dWr);
  MOE_CHECK_LAUNCH("router_wgrad_reduce");
  return MOE_OK;
}
