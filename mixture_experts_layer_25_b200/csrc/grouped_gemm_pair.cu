// Weight-gradient grouped GEMM on SM pairs (tcgen05 cta_group::2).
//
// Olmo-core 3 オープン混合エキスパート学習インフラストラクチャ, section
// "ルーティングと計算の最適化": the per-expert matmuls as one grouped GEMM;
// here the backward's weight gradients dW[e] = A_e^T dC_e, reduced over the
// rows of expert e's group.
//
// A cluster of two CTAs (two SMs) computes one 256 x 256 output tile with
// one MMA stream: each CTA loads the 128 output rows (M) of its half of A
// and the 128 output columns of its half of B into its own shared memory,
// the leader (cluster rank 0) issues tcgen05.mma.cta_group::2 over both
// halves, and each CTA's TMEM receives the accumulator rows of its own A
// half.  Per SM and K step that is 32 KB of operands for the work a 1-SM
// 128 x 256 tile does with 48 KB, so the ring holds six stages.
//
// Protocol (all waits bounded; a wait that gives up raises MOE_DEV_TIMEOUT):
//  * full[s] of the leader counts both CTAs' TMA bytes (its producer posts
//    the expected total; both producers' loads signal it with cta_group::2);
//  * the leader's MMA commits release empty[s] and fill acc_full[a] in both
//    CTAs at once (multicast commit);
//  * both CTAs' epilogue warps release acc_empty[a] of the leader;
//  * both CTAs allocate and free TMEM together (warp 1, same slot) and meet
//    at a cluster barrier before freeing it.
// No TMA load uses cluster multicast; every load reads this GPU's memory.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"

namespace moe {
namespace gp {

using namespace sm100;

constexpr int BM = 128;             // output rows per CTA (256 per pair)
constexpr int BN = 256;             // output columns per pair tile (128 of B per CTA)
constexpr int BK = 64;              // K (group rows) per stage
constexpr int MMA_K = 16;
constexpr int KSTEPS = BK / MMA_K;
constexpr int STAGES = 6;
constexpr int NUM_EPI_WARPS = 8;
constexpr int NUM_THREADS = 64 + 32 * NUM_EPI_WARPS;
constexpr int CHUNK = 32;
constexpr int BOX_BYTES = 32 * CHUNK * 2;
constexpr int A_BYTES = BM * BK * 2;              // 16 KB: two 64-column chunks of 64 rows
constexpr int B_BYTES = (BN / 2) * BK * 2;        // 16 KB: this CTA's 128 columns
constexpr int CHUNK_BYTES = BK * 128;             // one 64-column MN-major chunk (8 KB)
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int MAX_E = 1024;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + NUM_EPI_WARPS * BOX_BYTES;

struct Params {
  const int32_t* poff;
  const int32_t* offsets;   // unpadded group offsets (E + 1) or null (use poff)
  int E;
  int m_tiles;              // pair tiles along M (K_out / 256)
  int n_tiles;              // tiles along N (Ncols / 256)
  int k_out;                // output rows per expert (K_out)
  int n_split;              // > 0: columns >= n_split go to the second output
  int32_t* status;
};

__device__ __forceinline__ uint32_t bf16x2(float a, float b) { return pack2(a, b); }

// byte offset of 16-byte chunk j of row r inside a [32 rows x 64 B] box
// stored with the 64-byte swizzle
__device__ __forceinline__ uint32_t sw64(int r, int j) {
  return (uint32_t)(r * 64 + ((j ^ ((r >> 1) & 3)) << 4));
}

// instruction descriptor: bf16 x bf16 -> fp32, A and B MN-major, M = 256
// (the pair), N = 256
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                            ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);

__global__ void __launch_bounds__(NUM_THREADS, 1)
wgrad_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmC2,
                  const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES], empty_bar[STAGES];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], drain_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int poff_s[MAX_E + 1];
  __shared__ int krows_s[MAX_E];
  __shared__ int order_s[MAX_E];     // experts by descending reduction rows
  __shared__ volatile int abort_flag;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint8_t* sStg = sB + STAGES * B_BYTES;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = (int)cluster_id_x(), npairs = (int)nclusters_x();

  for (int i = threadIdx.x; i <= p.E; i += NUM_THREADS) poff_s[i] = p.poff[i];
  for (int e = threadIdx.x; e < p.E; e += NUM_THREADS)
    krows_s[e] = p.offsets ? p.offsets[e + 1] - p.offsets[e] : p.poff[e + 1] - p.poff[e];
  __syncthreads();
  // longest groups first: the pairs take tiles round-robin, so hot experts'
  // long reductions start at once instead of trailing (same order in every
  // CTA; ties by expert index)
  for (int e = threadIdx.x; e < p.E; e += NUM_THREADS) {
    const int ke = krows_s[e];
    int r = 0;
    for (int f = 0; f < p.E; ++f) {
      const int kf = krows_s[f];
      r += (kf > ke) || (kf == ke && f < e);
    }
    order_s[r] = e;
  }
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 2 * NUM_EPI_WARPS);
    }
    mbar_init(&drain_bar, 1);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch(&tmA);
    tma_prefetch(&tmB);
    tma_prefetch(&tmC);
    if (p.n_split > 0) tma_prefetch(&tmC2);
  }
  if (warp == 1) {
    tmem_alloc_pair(&tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();       // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;

  const int per_e = p.m_tiles * p.n_tiles;
  const int total = p.E * per_e;
  // pair tile -> expert, row-half origin m0 of this CTA, column tile nt
  auto decode = [&](int tile, int& e, int& m0, int& nt) {
    const int i = tile / per_e;
    e = order_s[i];
    const int rem = tile - i * per_e;
    const int mt = rem / p.n_tiles;
    nt = rem - mt * p.n_tiles;
    m0 = mt * 2 * BM + (int)rank * BM;
  };
  auto nkb_of = [&](int e) { return (krows_s[e] + BK - 1) / BK; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // lane 0 owns the barriers and issues both operands' loads
    const uint32_t full_leader0 = map_to_rank(&full_bar[0], 0);
    int stage = 0;
    uint32_t phase = 0;
    uint32_t used = 0, last_parity = 0;
    bool stop = false;
    for (int tile = pair; tile < total && !stop; tile += npairs) {
      int e, m0, nt;
      decode(tile, e, m0, nt);
      const int nkb = nkb_of(e);
      const int krow0 = poff_s[e];
      for (int kb = 0; kb < nkb; ++kb) {
        int ok = 1;
        if (lane == 0)
          ok = mbar_wait(&empty_bar[stage], phase ^ 1, &abort_flag, p.status, kWaitLimitNs);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) { stop = true; break; }
        const uint32_t fb = full_leader0 + (uint32_t)(stage * sizeof(uint64_t));
        if (leader && lane == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * STAGE_BYTES);
        __syncwarp();
        uint8_t* a_dst = sA + stage * A_BYTES;
        uint8_t* b_dst = sB + stage * B_BYTES;
        if (lane == 0) {
          tma_load_3d_pair(a_dst, &tmA, fb, 0, krow0 + kb * BK, m0 / 64);
          tma_load_3d_pair(b_dst, &tmB, fb, 0, krow0 + kb * BK, (nt * BN + (int)rank * (BN / 2)) / 64);
        }
        used |= 1u << stage;
        last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
    // the leader's full barriers count both CTAs' bytes: once the last phase
    // of every used stage has completed, every load of the pair has landed
    if (leader && lane == 0)
      for (int s = 0; s < STAGES; ++s)
        if (used & (1u << s)) {
          volatile int no_abort = 0;
          mbar_wait(&full_bar[s], (last_parity >> s) & 1, &no_abort, p.status, kWaitLimitNs);
        }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issue (leader only)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
      const uint32_t peer_acc_full0 = map_to_rank(&acc_full[0], 1);
      for (int tile = pair; tile < total && !abort_flag; tile += npairs, ++it) {
        int e, m0, nt;
        decode(tile, e, m0, nt);
        const int nkb = nkb_of(e);
        const int acc = it & 1;
        const uint32_t acc_par = (it >> 1) & 1;
        if (!mbar_wait(&acc_empty[acc], acc_par ^ 1, &abort_flag, p.status, kWaitLimitNs)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * 256;
        // K steps of the group's last block that hold real rows
        const int last_ks = nkb > 0 ? (krows_s[e] - (nkb - 1) * BK + MMA_K - 1) / MMA_K : 0;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, &abort_flag, p.status, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = a_base + stage * A_BYTES, sb = b_base + stage * B_BYTES;
#pragma unroll
          for (int ks = 0; ks < KSTEPS; ++ks) {
            if (kb == nkb - 1 && ks >= last_ks) break;
            const uint64_t ad = smem_desc(sa + ks * MMA_K * 128, CHUNK_BYTES, 1024, 2);
            const uint64_t bd = smem_desc(sb + ks * MMA_K * 128, CHUNK_BYTES, 1024, 2);
            mma_bf16_pair(d_tmem, ad, bd, kIdesc, (kb > 0 || ks > 0) ? 1u : 0u);
          }
          mma_commit_pair(&empty_bar[stage], 0x3);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (nkb > 0) {
          mma_commit_pair(&acc_full[acc], 0x3);
        } else {                         // empty group: both epilogues write zeros
          mbar_arrive(&acc_full[acc]);
          mbar_arrive_cluster(peer_acc_full0 + (uint32_t)(acc * sizeof(uint64_t)));
        }
      }
      // every MMA has completed (in both CTAs' view) before TMEM is freed
      mma_commit_pair(&drain_bar, 0x3);
    }
    if (lane == 0) {
      volatile int no_abort = 0;
      mbar_wait(&drain_bar, 0, &no_abort, p.status, kWaitLimitNs);
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM lane quarter
    const int ew = warp - 2;
    const int hc = ew >> 2;                 // half of the tile's 256 columns
    const int r = lane;
    uint8_t* stg = sStg + ew * BOX_BYTES;
    const uint32_t leader_acc_empty0 = map_to_rank(&acc_empty[0], 0);
    int it = 0;
    for (int tile = pair; tile < total; tile += npairs, ++it) {
      int e, m0, nt;
      decode(tile, e, m0, nt);
      const bool empty = nkb_of(e) <= 0;
      const int acc = it & 1;
      const uint32_t acc_par = (it >> 1) & 1;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&acc_full[acc], acc_par, &abort_flag, p.status, kWaitLimitNs);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * 256;
      const int n0 = nt * BN;
      const CUtensorMap* map = &tmC;
      int x0 = n0;
      if (p.n_split > 0 && n0 >= p.n_split) { map = &tmC2; x0 = n0 - p.n_split; }
      const int y0 = e * p.k_out + m0 + q * 32;
      uint32_t av[32];
#pragma unroll 1
      for (int ci = 0; ci < 4; ++ci) {
        const int c = hc * (BN / 2) + ci * CHUNK;
        if (!empty) {
          tmem_ld32(tbase + c, av);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) av[i] = 0u;
        }
        if (lane == 0) bulk_wait_read<0>();      // the box's previous store has read it
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 w;
          w.x = bf16x2(__uint_as_float(av[8 * j + 0]), __uint_as_float(av[8 * j + 1]));
          w.y = bf16x2(__uint_as_float(av[8 * j + 2]), __uint_as_float(av[8 * j + 3]));
          w.z = bf16x2(__uint_as_float(av[8 * j + 4]), __uint_as_float(av[8 * j + 5]));
          w.w = bf16x2(__uint_as_float(av[8 * j + 6]), __uint_as_float(av[8 * j + 7]));
          *reinterpret_cast<uint4*>(stg + sw64(r, j)) = w;
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(map, stg, x0 + c, y0);
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {                          // release the accumulator to the leader's MMA
        if (leader) mbar_arrive(&acc_empty[acc]);
        else mbar_arrive_cluster(leader_acc_empty0 + (uint32_t)(acc * sizeof(uint64_t)));
      }
    }
    if (lane == 0) bulk_wait_all();
  }

  // after an abort, loads of the pair may still be in flight with no phase
  // left to wait on: give them time to land before shared memory is released
  if (abort_flag) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 100000ull) {
    }
  }
  // every warp reconverges first: lanes that skipped a one-lane role loop
  // (producer, MMA issue) must not reach the cluster barrier, or the warp-wide
  // TMEM free after it, ahead of that lane
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

// 3-D MN-major view: (128-byte chunk, rows, chunk index) of a row-major
// bf16 [rows, cols] array; box (64, box_rows, nchunk)
bool map_mn3(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows,
             uint32_t nchunk) {
  auto fn = tensor_map_encoder();
  if (!fn || cols % 64) return false;
  cuuint64_t dims[3] = {64, rows, cols / 64};
  cuuint64_t strides[2] = {cols * 2, 128};
  cuuint32_t box[3] = {64, box_rows, nchunk};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
            uint32_t box_outer, CUtensorMapSwizzle swz) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

moe_status_t launch(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c,
                    const CUtensorMap& c2, const Params& p, int tiles, cudaStream_t s) {
  auto kern = wgrad_pair_kernel;
  MOE_TRY(set_smem_limit(reinterpret_cast<const void*>(kern), SMEM, "wgrad_pair"));
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // one pair per co-resident cluster slot (persistent), at most one per tile
  cfg.gridDim = dim3(2, 1, 1);
  int max_clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg) != cudaSuccess || max_clusters < 1)
    max_clusters = num_sms() / 2;
  const int pairs = std::max(1, std::min(max_clusters, tiles));
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a, b, c, c2, p);
  if (e != cudaSuccess) {
    count_launch();
    set_error("wgrad_pair: launch: %s", cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  MOE_CHECK_LAUNCH("wgrad_pair");
  return MOE_OK;
}

}  // namespace gp

// Weight-gradient grouped GEMM (BF16) on SM pairs: dB[e] = A_e^T dC_e (and
// dB3 from dC's second half when dB3 is given), reduced over the rows of
// group e up to its last real row (offsets, or every padded row).  A is the
// padded buffer [A_pad_max, K].  K % 256 == 0, N % 256 == 0.
moe_status_t grouped_gemm_wgrad_pair(const void* A, const void* dC, const int32_t* poff,
                                     const int32_t* offsets,
                                     int E, int A_pad_max, int K, int N, void* dB, void* dB3,
                                     int32_t* dev_status, cudaStream_t s) {
  using namespace gp;
  MOE_CHECK_ARG(E > 0 && E <= MAX_E, "wgrad_pair: E must be in [1, %d]", MAX_E);
  MOE_CHECK_ARG(A_pad_max > 0 && A_pad_max % 128 == 0, "wgrad_pair: A_pad_max %% 128");
  MOE_CHECK_ARG(K > 0 && K % 256 == 0 && N > 0 && N % 256 == 0, "wgrad_pair: K, N %% 256");
  MOE_CHECK_ARG(A && dC && dB && poff, "wgrad_pair: null pointer");
  const int Ncols = dB3 ? 2 * N : N;
  Params p{};
  p.poff = poff;
  p.offsets = offsets;
  p.E = E;
  p.m_tiles = K / 256;
  p.n_tiles = Ncols / BN;
  p.k_out = K;
  p.n_split = dB3 ? N : 0;
  p.status = dev_status;
  CUtensorMap ma, mb, mc, mc2;
  bool ok = map_mn3(&ma, A, K, A_pad_max, BK, 2);
  ok = ok && map_mn3(&mb, dC, Ncols, A_pad_max, BK, 2);
  ok = ok && map_2d(&mc, dB, N, (uint64_t)E * K, CHUNK, 32, CU_TENSOR_MAP_SWIZZLE_64B);
  ok = ok && (dB3 ? map_2d(&mc2, dB3, N, (uint64_t)E * K, CHUNK, 32, CU_TENSOR_MAP_SWIZZLE_64B)
                  : (mc2 = mc, true));
  if (!ok) {
    set_error("wgrad_pair: tensor map encoding failed");
    return MOE_ERR_CUDA;
  }
  const int tiles = E * p.m_tiles * p.n_tiles;
  return launch(ma, mb, mc, mc2, p, tiles, s);
}

}  // namespace moe
