// Grouped GEMM with the tokens on the MMA's N side ("tokens-N"), BF16.
//
// Olmo-core 3 オープン混合エキスパート学習インフラストラクチャ, section
// "ルーティングと計算の最適化": the per-expert matmuls of the expert feed-forward
// run as one grouped GEMM over the expert-contiguous buffers.
//
// The tiles of the main grouped GEMM put 128 tokens on the MMA's M side, so
// the zero rows that pad every expert group to a multiple of 128 are
// multiplied like real rows (13% of the rows at T = 16384, E = 128, k = 4).
// Here the weights are the M side (128 output features per tile) and the
// tokens the N side: N may be any multiple of 16 up to 256, so an expert's
// real rows are split evenly over ceil(rows / 256) token blocks (each a
// multiple of 32 rows) and only the rows that exist are multiplied.
//
//  * persistent CTAs, 320 threads: TMA producer warp, MMA warp (one thread,
//    owns 512 TMEM columns = two 128 x 256 fp32 accumulators), 8 epilogue
//    warps (two per TMEM lane quarter; each takes half of the token columns).
//  * accumulator D[feature, token]: the epilogue thread of TMEM lane f holds
//    one output feature for 32 tokens per tcgen05.ld and writes them down a
//    column of a 32 x 32 shared-memory box (64-byte swizzle), which a TMA
//    bulk store puts into the row-major output [rows, features].
//  * output rows from the group's last real row to its padded end are
//    written as zeros (from a zero box), so every padded output row is
//    defined as before.
//  * SwiGLU: a tile's 128 weight rows are 64 features of W1 followed by the
//    same 64 features of W3; the W3 warps hand their bf16 H3 box to the W1
//    warps of the same lanes and token half through shared memory, so h is
//    formed from the stored bf16 H3 (the value the backward reads).
//  * every mbarrier wait is bounded (status word, clean exit), as in the
//    main grouped GEMM.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"

namespace moe {
namespace tn {

using namespace sm100;

constexpr int BM = 128;                 // output features per tile (MMA M)
constexpr int BNMAX = 256;              // tokens per tile at most (MMA N)
constexpr int BK = 64;                  // K per stage (bf16, 128-byte rows)
constexpr int MMA_K = 16;
constexpr int KSTEPS = BK / MMA_K;
constexpr int STAGES = 4;
constexpr int NUM_EPI_WARPS = 8;
constexpr int NUM_THREADS = 64 + 32 * NUM_EPI_WARPS;
constexpr int A_BYTES = BM * 128;       // weights: 128 rows x 128 bytes of K
constexpr int B_BYTES = BNMAX * 128;    // tokens: 256 rows x 128 bytes of K
constexpr int CHUNK_BYTES = BK * 128;   // one 64-feature chunk of an MN-major weight tile
constexpr int BOX_BYTES = 32 * 64;      // 32 tokens x 32 features, bf16
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int MAX_E = 1024;

enum Epi { TN_STORE = 0, TN_SWIGLU = 1 };
enum ALoad { A_MN = 0, A_K = 1, A_K_DUAL = 2 };

struct Params {
  const int32_t* poff;      // padded group offsets (E + 1)
  const int32_t* offsets;   // unpadded group offsets (E + 1), or null: all padded rows are real
  int E;
  int n_fb;                 // feature blocks per token block
  int num_kb;               // K blocks
  int k_split;              // A_K_DUAL: first K index taken from the second weight
  int a_rows_per_e;         // rows of the weight map per expert
  int feat_per_fb;          // output features per feature block (128; SwiGLU: 64)
  int half;                 // SwiGLU: H3 column offset in aux (= F)
  const float* row_scale;   // STORE: optional rank-1 term row_scale[row] * col_vec[e * col_ld + n]
  const float* col_vec;
  int col_ld;
  int32_t* status;
};

// byte offset of element (token j, feature i) inside a [32 tokens x 32
// features] bf16 box stored with the 64-byte swizzle
__device__ __forceinline__ uint32_t box_off(int j, int i) {
  return (uint32_t)(j * 64 + ((((i >> 3) ^ (j >> 1)) & 3) << 4) + ((i & 7) << 1));
}

__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// barrier over n threads that also ANDs a predicate across them
__device__ __forceinline__ bool named_bar_and(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ uint32_t idesc_bf16(bool a_mn, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

// silu(z) = z sigmoid(z) with the 2-ulp fast division (as the rows-mode kernels)
__device__ __forceinline__ float silu_f(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

struct Tile {
  int e, fb;
  int start;      // first row of the token block
  int n_real;     // real rows in the block
  int n_mma;      // MMA N: n_real rounded up to 16
  int store;      // rows this tile writes: the block, plus the padding after the group's last real row
};

template <int EPI, int ALOAD>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_tn_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmW3,
               const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC,
               const __grid_constant__ CUtensorMap tmAux, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES], empty_bar[STAGES];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], drain_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;                                    // STAGES x A_BYTES
  uint8_t* sB = sA + STAGES * A_BYTES;                   // STAGES x B_BYTES
  uint8_t* sStg = sB + STAGES * B_BYTES;                 // one box per epilogue warp
  uint8_t* sZero = sStg + NUM_EPI_WARPS * BOX_BYTES;     // a box of zeros
  int* poff_s = reinterpret_cast<int*>(sZero + BOX_BYTES);   // [E + 1]
  int* cnt_s = poff_s + (p.E + 1);                           // [E] real rows
  int* tb_s = cnt_s + (p.E + 1);                             // [E + 1] token-block prefix

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int i = threadIdx.x; i <= p.E; i += NUM_THREADS) poff_s[i] = p.poff[i];
  for (int i = threadIdx.x; i < p.E; i += NUM_THREADS)
    cnt_s[i] = p.offsets ? p.offsets[i + 1] - p.offsets[i] : p.poff[i + 1] - p.poff[i];
  for (int i = threadIdx.x; i < BOX_BYTES / 16; i += NUM_THREADS)
    reinterpret_cast<uint4*>(sZero)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], NUM_EPI_WARPS);
    }
    mbar_init(&drain_bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == 0) {
    // token blocks per expert, prefix over the experts (one warp scan)
    int carry = 0;
    for (int base = 0; base < p.E; base += 32) {
      const int e = base + lane;
      const int c = e < p.E ? cnt_s[e] : 0;
      int nb = (c + BNMAX - 1) / BNMAX;
      int incl = nb;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (e < p.E) tb_s[e] = carry + incl - nb;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) tb_s[p.E] = carry;
    if (lane == 0) {
      tma_prefetch(&tmW);
      if (ALOAD == A_K_DUAL || EPI == TN_SWIGLU) tma_prefetch(&tmW3);
      tma_prefetch(&tmX);
      tma_prefetch(&tmC);
      if (EPI == TN_SWIGLU) tma_prefetch(&tmAux);
    }
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  const int total = tb_s[p.E] * p.n_fb;

  auto decode = [&](int tile) {
    Tile t;
    const int tb = tile / p.n_fb;
    t.fb = tile - tb * p.n_fb;
    int lo = 0, hi = p.E - 1;            // largest e with tb_s[e] <= tb
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tb_s[mid] <= tb) lo = mid; else hi = mid - 1;
    }
    t.e = lo;
    const int c = cnt_s[lo];
    const int nb = (c + BNMAX - 1) / BNMAX;
    const int b = tb - tb_s[lo];
    const int bs = (((c + nb - 1) / nb) + 31) & ~31;   // block size, a multiple of 32
    const int r0 = b * bs;
    t.start = poff_s[lo] + r0;
    t.n_real = min(bs, c - r0);
    t.n_mma = (t.n_real + 15) & ~15;
    const bool last = b == nb - 1;
    t.store = last ? poff_s[lo + 1] - t.start : bs;
    return t;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t used = 0, last_parity = 0;
      for (int tile = blockIdx.x; tile < total && !abort_flag; tile += gridDim.x) {
        const Tile t = decode(tile);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_flag, p.status, kWaitLimitNs)) break;
          uint64_t* fb = &full_bar[stage];
          mbar_arrive_expect_tx(fb, A_BYTES + B_BYTES);
          uint8_t* a_dst = sA + stage * A_BYTES;
          const int wrow = t.e * p.a_rows_per_e;
          if constexpr (ALOAD == A_MN) {
            // weights [K rows, features]: two 64-feature chunks
            if constexpr (EPI == TN_SWIGLU) {
              const int f0 = t.fb * 64;
              tma_load_2d(a_dst, &tmW, fb, f0, wrow + kb * BK);
              tma_load_2d(a_dst + CHUNK_BYTES, &tmW3, fb, f0, wrow + kb * BK);
            } else {
              const int f0 = t.fb * BM;
              tma_load_2d(a_dst, &tmW, fb, f0, wrow + kb * BK);
              tma_load_2d(a_dst + CHUNK_BYTES, &tmW, fb, f0 + 64, wrow + kb * BK);
            }
          } else if constexpr (ALOAD == A_K) {
            tma_load_2d(a_dst, &tmW, fb, kb * BK, wrow + t.fb * BM);
          } else {
            const int k = kb * BK;
            if (k < p.k_split) tma_load_2d(a_dst, &tmW, fb, k, wrow + t.fb * BM);
            else tma_load_2d(a_dst, &tmW3, fb, k - p.k_split, wrow + t.fb * BM);
          }
          tma_load_2d(sB + stage * B_BYTES, &tmX, fb, kb * BK, t.start);
          used |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      for (int s = 0; s < STAGES; ++s)
        if (used & (1u << s)) {
          volatile int no_abort = 0;
          mbar_wait(&full_bar[s], (last_parity >> s) & 1, &no_abort, p.status, kWaitLimitNs);
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issue
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
      for (int tile = blockIdx.x; tile < total && !abort_flag; tile += gridDim.x, ++it) {
        const Tile t = decode(tile);
        const uint32_t idesc = idesc_bf16(ALOAD == A_MN, t.n_mma);
        const int acc = it & 1;
        const uint32_t acc_par = (it >> 1) & 1;
        if (!mbar_wait(&acc_empty[acc], acc_par ^ 1, &abort_flag, p.status, kWaitLimitNs)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * 256;
        bool ok = true;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, &abort_flag, p.status, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = a_base + stage * A_BYTES, sb = b_base + stage * B_BYTES;
#pragma unroll
          for (int ks = 0; ks < KSTEPS; ++ks) {
            uint64_t ad;
            if constexpr (ALOAD == A_MN) ad = smem_desc(sa + ks * MMA_K * 128, CHUNK_BYTES, 1024, 2);
            else ad = smem_desc(sa + ks * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(sb + ks * 32, 16, 1024, 2);
            mma_bf16(d_tmem, ad, bd, idesc, (kb > 0 || ks > 0) ? 1u : 0u);
          }
          mma_commit(&empty_bar[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        mma_commit(&acc_full[acc]);
      }
      mma_commit(&drain_bar);
      volatile int no_abort = 0;
      mbar_wait(&drain_bar, 0, &no_abort, p.status, kWaitLimitNs);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM lane quarter
    const int ew = warp - 2;                // 0..7
    const int hc = ew >> 2;                 // token half of the tile
    uint8_t* box = sStg + ew * BOX_BYTES;
    // SwiGLU: warps of quarters 2, 3 (W3 features) hand their H3 box to the
    // warps of quarters 0, 1 (W1 features) of the same token half
    const int pair_q = q & 1;
    const int bar_id = 1 + pair_q + 2 * hc;
    const bool is_u = EPI == TN_SWIGLU && q >= 2;
    // epilogue warp of quarter q' and half hc is ew = 4 hc + (q' ^ 2), so the
    // W3 partner (quarter q ^ 2) of a W1 warp owns box 4 hc + q
    uint8_t* pbox = sStg + (hc * 4 + q) * BOX_BYTES;
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      const Tile t = decode(tile);
      const int acc = it & 1;
      const uint32_t acc_par = (it >> 1) & 1;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&acc_full[acc], acc_par, &abort_flag, p.status, kWaitLimitNs);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if constexpr (EPI == TN_SWIGLU) ok = named_bar_and(bar_id, 64, ok != 0 && !abort_flag);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * 256;
      const int fi = q * 32 + lane;                       // feature row of the tile
      // output column of this thread's feature
      int col;
      if constexpr (EPI == TN_SWIGLU) col = t.fb * 64 + (q & 1) * 32;   // + lane in the box
      else col = t.fb * BM + q * 32;
      float cval = 0.f;
      if constexpr (EPI == TN_STORE)
        if (p.row_scale) cval = p.col_vec[(size_t)t.e * p.col_ld + t.fb * BM + fi];

      // token chunks of 32 held in TMEM (columns [hc*128, hc*128 + 128))
#pragma unroll 1
      for (int ci = 0; ci < 4; ++ci) {
        const int c0 = hc * 128 + ci * 32;
        if (c0 >= t.store) break;                  // uniform for the pair
        const int y = t.start + c0;
        uint32_t v[32];
        if (c0 < t.n_mma) {
          tmem_ld32(tbase + c0, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0u;
        }
        const int nv = t.n_real - c0;              // columns with real tokens in this chunk
        if constexpr (EPI == TN_STORE) {
          if (lane == 0) bulk_wait_read<0>();
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float a = j < nv ? __uint_as_float(v[j]) : 0.f;
            if (p.row_scale && j < nv) a = fmaf(p.row_scale[y + j], cval, a);
            *reinterpret_cast<__nv_bfloat16*>(box + box_off(j, lane)) = __float2bfloat16_rn(a);
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmC, box, col, y);
            bulk_commit();
          }
        } else {
          if (is_u) {
            // H3 box (bf16), stored and handed to the partner
            if (lane == 0) bulk_wait_read<0>();
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 32; ++j)
              *reinterpret_cast<__nv_bfloat16*>(box + box_off(j, lane)) =
                  __float2bfloat16_rn(j < nv ? __uint_as_float(v[j]) : 0.f);
            fence_async_smem();
            named_bar_sync(bar_id, 64);              // box ready
            if (lane == 0) {
              tma_store_2d(&tmAux, box, p.half + col, y);
              bulk_commit();
            }
            named_bar_sync(bar_id, 64);              // partner has read it
          } else {
            float h[32];
            named_bar_sync(bar_id, 64);              // partner's H3 box ready
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float u = __bfloat162float(
                  *reinterpret_cast<const __nv_bfloat16*>(pbox + box_off(j, lane)));
              h[j] = j < nv ? silu_f(__uint_as_float(v[j])) * u : 0.f;
            }
            named_bar_sync(bar_id, 64);
            // h, then H1, through this warp's box
            if (lane == 0) bulk_wait_read<0>();
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 32; ++j)
              *reinterpret_cast<__nv_bfloat16*>(box + box_off(j, lane)) = __float2bfloat16_rn(h[j]);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmC, box, col, y);
              bulk_commit();
              bulk_wait_read<0>();
            }
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 32; ++j)
              *reinterpret_cast<__nv_bfloat16*>(box + box_off(j, lane)) =
                  __float2bfloat16_rn(j < nv ? __uint_as_float(v[j]) : 0.f);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmAux, box, col, y);
              bulk_commit();
            }
          }
        }
      }
      // padding rows past TMEM's 256 columns: zero boxes
      if (lane == 0) {
        for (int c0 = BNMAX + hc * 32; c0 < t.store; c0 += 64) {
          const int y = t.start + c0;
          if constexpr (EPI == TN_STORE) {
            tma_store_2d(&tmC, sZero, col, y);
          } else if (is_u) {
            tma_store_2d(&tmAux, sZero, p.half + col, y);
          } else {
            tma_store_2d(&tmC, sZero, col, y);
            tma_store_2d(&tmAux, sZero, col, y);
          }
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
    }
    if (lane == 0) bulk_wait_all();
  }

  // every warp reconverges first: lanes that skipped a one-lane role loop
  // (producer, MMA issue) must not reach the CTA barrier, or the warp-wide
  // TMEM free after it, ahead of that lane
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ----------------------------------------------------------------- host side
// 2-D map over a row-major [outer, inner] bf16 array, box {box_inner, box_outer}
moe_status_t map2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                   uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  auto fn = tensor_map_encoder();
  if (!fn) {
    set_error("cuTensorMapEncodeTiled unavailable");
    return MOE_ERR_CUDA;
  }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("gemm_tn: cuTensorMapEncodeTiled failed (%d): %llu x %llu box %u x %u", (int)r,
              (unsigned long long)inner, (unsigned long long)outer, box_inner, box_outer);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

size_t smem_bytes(int E) {
  return 1024 + (size_t)STAGES * (A_BYTES + B_BYTES) + (size_t)(NUM_EPI_WARPS + 1) * BOX_BYTES +
         (size_t)3 * (E + 1) * sizeof(int);
}

template <int EPI, int ALOAD>
moe_status_t launch(const CUtensorMap& w, const CUtensorMap& w3, const CUtensorMap& x,
                    const CUtensorMap& c, const CUtensorMap& aux, const Params& p, int max_tiles,
                    cudaStream_t s) {
  auto kern = gemm_tn_kernel<EPI, ALOAD>;
  const size_t smem = smem_bytes(p.E);
  MOE_TRY(set_smem_limit(reinterpret_cast<const void*>(kern), smem, "gemm_tn"));
  const int grid = std::max(1, std::min(num_sms(), max_tiles));
  kern<<<grid, NUM_THREADS, smem, s>>>(w, w3, x, c, aux, p);
  MOE_CHECK_LAUNCH("gemm_tn");
  return MOE_OK;
}

}  // namespace tn

using namespace tn;

// Tokens-N grouped GEMM (BF16), three forms:
//  * epilogue MOE_EPI_SWIGLU: X [A_pad, K] times W [E, K, N] and W3 (same
//    shape; weights MN-major) -> h = silu(X W) * bf16(X W3) [A_pad, N] and
//    aux = [X W | X W3] [A_pad, 2N];
//  * MOE_EPI_NONE, W3 == null: C = X W [A_pad, N] (weights MN-major);
//  * MOE_EPI_NONE, w_kmajor: C = X[:, :K/2] W^T + X[:, K/2:] W3^T with W, W3
//    [E, N, K/2] (dgrad of the dual GEMM; W3 may be null for a single K),
//    plus the optional rank-1 term row_scale[row] * col_vec[e * N + n].
// offsets (unpadded group offsets) or null (every padded row counts).
moe_status_t gemm_tn(int epilogue, const void* X, const void* W, const void* W3, int w_kmajor,
                     const int32_t* poff, const int32_t* offsets, int E, int A_pad_max, int N,
                     int K, void* C, void* aux, const float* row_scale, const float* col_vec,
                     int32_t* dev_status, cudaStream_t s) {
  MOE_CHECK_ARG(E > 0 && E <= MAX_E, "gemm_tn: E must be in [1, %d]", MAX_E);
  MOE_CHECK_ARG(A_pad_max > 0 && A_pad_max % 128 == 0, "gemm_tn: A_pad_max %% 128");
  MOE_CHECK_ARG(X && W && C && poff, "gemm_tn: null pointer");
  MOE_CHECK_ARG(K > 0 && K % BK == 0, "gemm_tn: K %% %d", BK);
  MOE_CHECK_ARG((row_scale == nullptr) == (col_vec == nullptr) && (!col_vec || aligned16(col_vec)),
                "gemm_tn: row_scale and col_vec go together");
  // every argument is checked before the first driver call
  if (epilogue == MOE_EPI_SWIGLU) {
    MOE_CHECK_ARG(W3 && aux && !w_kmajor && N % 64 == 0 && !row_scale,
                  "gemm_tn: SwiGLU needs W3, aux, MN-major weights and N %% 64");
  } else {
    MOE_CHECK_ARG(epilogue == MOE_EPI_NONE, "gemm_tn: epilogue must be NONE or SWIGLU");
    MOE_CHECK_ARG(N % BM == 0, "gemm_tn: N %% %d", BM);
    MOE_CHECK_ARG(w_kmajor || (!W3 && !row_scale),
                  "gemm_tn: MN-major weights take neither W3 nor a rank-1 term");
    MOE_CHECK_ARG(!w_kmajor || (W3 ? K / 2 : K) % BK == 0, "gemm_tn: K per weight %% %d", BK);
  }
  Params p{};
  p.poff = poff;
  p.offsets = offsets;
  p.E = E;
  p.num_kb = K / BK;
  p.status = dev_status;
  p.row_scale = row_scale;
  p.col_vec = col_vec;
  p.col_ld = N;
  CUtensorMap mw, mw3, mx, mc, maux;
  MOE_TRY(map2d(&mx, X, K, A_pad_max, BK, BNMAX, CU_TENSOR_MAP_SWIZZLE_128B));
  MOE_TRY(map2d(&mc, C, N, A_pad_max, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B));
  if (epilogue == MOE_EPI_SWIGLU) {
    p.n_fb = N / 64;
    p.feat_per_fb = 64;
    p.a_rows_per_e = K;
    p.half = N;
    MOE_TRY(map2d(&mw, W, N, (uint64_t)E * K, 64, BK, CU_TENSOR_MAP_SWIZZLE_128B));
    MOE_TRY(map2d(&mw3, W3, N, (uint64_t)E * K, 64, BK, CU_TENSOR_MAP_SWIZZLE_128B));
    MOE_TRY(map2d(&maux, aux, 2ULL * N, A_pad_max, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B));
    const int max_tiles = (A_pad_max / 32) * p.n_fb;
    return launch<TN_SWIGLU, A_MN>(mw, mw3, mx, mc, maux, p, max_tiles, s);
  }
  p.n_fb = N / BM;
  p.feat_per_fb = BM;
  const int max_tiles = (A_pad_max / 32) * p.n_fb;
  if (!w_kmajor) {
    p.a_rows_per_e = K;
    MOE_TRY(map2d(&mw, W, N, (uint64_t)E * K, 64, BK, CU_TENSOR_MAP_SWIZZLE_128B));
    return launch<TN_STORE, A_MN>(mw, mw, mx, mc, mc, p, max_tiles, s);
  }
  const int Kw = W3 ? K / 2 : K;          // K columns of each weight
  p.a_rows_per_e = N;
  p.k_split = Kw;
  MOE_TRY(map2d(&mw, W, Kw, (uint64_t)E * N, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B));
  if (!W3) return launch<TN_STORE, A_K>(mw, mw, mx, mc, mc, p, max_tiles, s);
  MOE_TRY(map2d(&mw3, W3, Kw, (uint64_t)E * N, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B));
  return launch<TN_STORE, A_K_DUAL>(mw, mw3, mx, mc, mc, p, max_tiles, s);
}

}  // namespace moe

extern "C" moe_status_t moe_grouped_gemm_tn(int epilogue, const void* X, const void* W,
                                            const void* W3, int w_kmajor, const int32_t* poff,
                                            const int32_t* offsets, int E, int A_pad_max, int N,
                                            int K, void* C, void* aux, const float* row_scale,
                                            const float* col_vec, int32_t* dev_status,
                                            moe_stream_t stream) {
  return moe::gemm_tn(epilogue, X, W, W3, w_kmajor, poff, offsets, E, A_pad_max, N, K, C, aux,
                      row_scale, col_vec, dev_status, reinterpret_cast<cudaStream_t>(stream));
}
