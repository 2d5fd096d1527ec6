// Grouped GEMM over expert groups on the 5th-generation tensor cores.
//
// Olmo-core 3 オープン混合エキスパート学習インフラストラクチャ, section
// "ルーティングと計算の最適化": the many small per-expert matmuls are batched
// into one grouped GEMM; section "MXFP8による精度最適化": MXFP8 for the expert
// feed-forward compute.
//
// Design (sm_100a):
//  * persistent CTAs (one per SM), 320 threads: warp 0 issues TMA loads,
//    warp 1 issues tcgen05.mma (one thread) and owns TMEM, warps 2..9 are
//    the epilogue: two per TMEM lane quarter (32 accumulator rows), one per
//    half of the tile's columns; each moves 32-column chunks TMEM ->
//    registers -> a 64-byte-swizzled shared-memory box -> TMA bulk store, so
//    global traffic is whole coalesced boxes.
//  * tile 128 x 256, fp32 accumulators in TMEM (two buffers for BF16, so the
//    epilogue of tile i overlaps the main loop of tile i+1), a 3- or 4-stage
//    shared-memory ring fed by TMA with 128-byte swizzle; MN-major operands
//    come through 3-D tensor maps (one TMA op per operand and stage).
//  * device-side tile schedule read from poff: "rows" mode walks the
//    128-row tiles of the expert-contiguous buffer (every group starts on a
//    multiple of 128, so a tile never mixes experts) times the N tiles;
//    "wgrad" mode walks (expert, M tile, N tile) and reduces over the rows
//    of the expert's group, stopping at its last real row.
//  * epilogues: plain store (+ an optional rank-1 term), SwiGLU (h, H1, H3),
//    SwiGLU backward, and the router's top-k / gates / ranks / histograms.
//  * every mbarrier wait is bounded; a wait that gives up raises
//    MOE_DEV_TIMEOUT in the caller's status word and the CTA drains and
//    exits.
//  * MXFP8: E4M3 operands with kind::mxf8f6f4.block_scale; the E8M0 scales
//    of each stage are bulk-copied to shared memory and moved into TMEM
//    with tcgen05.cp; one accumulator buffer (TMEM also holds the scales),
//    handed back to the MMA warp as soon as the epilogue has it in registers.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "mx.cuh"
#include "sm100.cuh"

namespace moe {
namespace gg {

using namespace sm100;

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int NUM_EPI_WARPS = 8;    // two per TMEM lane quarter, each half of the columns
constexpr int NUM_THREADS = 64 + 32 * NUM_EPI_WARPS;
constexpr int CHUNK = 32;           // epilogue columns per staged box
constexpr int BOX_BYTES = 32 * CHUNK * 2;   // 32 rows x 32 bf16
constexpr int A_BYTES = BM * 128;   // 128-byte rows (64 bf16 or 128 fp8 of K)
constexpr int B_BYTES = BN * 128;
constexpr int SFA_BYTES = 512;      // 128 rows x 4 scale bytes
constexpr int SFB_BYTES = 1024;     // 256 rows x 4 scale bytes
constexpr int MAX_E = 1024;
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s

enum Epi { EPI_STORE = 0, EPI_SWIGLU = 1, EPI_SWIGLU_BWD = 2, EPI_ROUTER = 3, EPI_ROUTER4 = 4 };
// the router epilogue keeps a running top-k of 8 slots (EPI_ROUTER, k <= 8)
// or 4 slots (EPI_ROUTER4, k <= 4)
__host__ __device__ constexpr bool is_router(int epi) { return epi == EPI_ROUTER || epi == EPI_ROUTER4; }

// pipeline depth and per-warp staging (boxes of 2 KB) for each epilogue,
// within the 227 KB of shared memory per CTA: STORE uses one box per warp
// with a 4-stage ring; SwiGLU stages h / H1 / H3; the SwiGLU backward
// double-buffers H1/H3 pairs (both with a 3-stage ring)
#ifndef MOE_GG_SWIGLU_STAGES
#define MOE_GG_SWIGLU_STAGES 4    // 4: one box, stores in turn; 3: h/H1/H3 boxes per warp
#endif
#ifndef MOE_GG_STORE_BOXES
#define MOE_GG_STORE_BOXES 1      // 1: 4-stage ring; 2: double-buffered boxes, 3 stages
#endif
#ifndef MOE_GG_WGRAD_BOXES
#define MOE_GG_WGRAD_BOXES 1      // weight-gradient tiles: 2 = double-buffered boxes, 3 stages
#endif
template <bool MX, int EPI, bool WGRAD = false> struct EpiCfg {
  static constexpr int SWIGLU_STAGES = MX ? 3 : MOE_GG_SWIGLU_STAGES;
  static constexpr int STORE_BOXES = WGRAD ? MOE_GG_WGRAD_BOXES : MOE_GG_STORE_BOXES;
  static constexpr int STAGES = EPI == EPI_STORE ? (STORE_BOXES == 1 ? 4 : 3)
                              : EPI == EPI_SWIGLU ? SWIGLU_STAGES
                              : is_router(EPI) ? 4 : 3;
  static constexpr int BOXES = EPI == EPI_STORE ? STORE_BOXES
                             : is_router(EPI) ? 1
                             : EPI == EPI_SWIGLU ? (SWIGLU_STAGES == 4 ? 1 : 3) : 4;
  static constexpr int STG = BOXES * BOX_BYTES;
  // the router stage holds two B tiles (one per weight split) of <= 128 columns
  static constexpr int B_STAGE = is_router(EPI) ? 2 * 128 * 128 : B_BYTES;
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * (A_BYTES + B_STAGE +
                                 (MX ? SFA_BYTES + SFB_BYTES : 0)) + NUM_EPI_WARPS * STG;
};

// byte offset of 16-byte chunk j of row r inside a [32 rows x 64 B] box
// stored with the 64-byte swizzle (chunk index XOR row bits 1..2)
__device__ __forceinline__ uint32_t sw64(int r, int j) {
  return (uint32_t)(r * 64 + ((j ^ ((r >> 1) & 3)) << 4));
}
enum BLoad { B_MN = 0, B_MN_DUAL_N = 1, B_K = 2, B_K_DUAL_K = 3 };

struct Params {
  const int32_t* poff;
  const int32_t* offsets;   // wgrad: unpadded group offsets (E + 1) or null (use poff)
  int E;
  int wgrad;          // 0: rows mode; 1: weight-gradient mode
  int n_tiles;        // tiles along N
  int m_tiles_w;      // wgrad: M tiles (K_out / 128)
  int num_kb;         // rows mode: K blocks per tile
  int b_rows_per_e;   // rows of the B tensor map per expert (rows mode)
  int k_split;        // B_K_DUAL_K: first K index taken from B3
  // MX scales (byte pointers into the tensor-core scale layout)
  const uint8_t* a_sc; int a_sc_kchunks;
  const uint8_t* b_sc; const uint8_t* b3_sc; int b_sc_kchunks;
  // epilogue
  __nv_bfloat16* C; long long ldc;
  __nv_bfloat16* C2; int n_split;
  __nv_bfloat16* aux; long long ld_aux; int half;
  long long c_expert_stride;
  // rows-mode STORE: optional rank-1 term C[row, n] += row_scale[row] * col_vec[e * col_ld + n]
  const float* row_scale; const float* col_vec; int col_ld;
  int k_out;          // wgrad: output rows per expert (K of the weight)
  // dense single-group mode (router): rows [0, dense_rows), no poff
  int dense_rows;
  int split_rows;     // router: rows per weight split in the B map (= d)
  int a3d, b3d;       // MN-major operand maps are 3-D (chunk, row, chunk index): one load per stage
  int mma_n;          // > 0: MMA N (multiple of 16, <= 256) instead of BN
  int b_boxes;        // > 0: MN-major B boxes loaded per stage (<= BN / chunk)
  // gathered A (GATHER kernels): row r of the padded A operand is row
  // a_src[r] of the unpermuted tokens (a_src[r] < 0: a zero row, read as the
  // out-of-range row a_oob)
  const int32_t* a_src; int a_oob;
  const __nv_bfloat16* a_x; int a_ld;   // the unpermuted rows and their length (K or M)
  // router epilogue
  const float* r_bias; float* r_logits; int32_t* r_topk; float* r_gates;
  int32_t* r_rank; int32_t* r_hist; int r_k; int r_E;
  // MXFP8 epilogues that quantise their bf16 output in place of storing it
  // (SwiGLU: h; SwiGLU backward: dA1 | dA3): codes along the row and down
  // the columns through the tmQr / tmQc maps, scale bytes in the
  // tensor-core layouts with K = the row length (q_row_kchunks = cols / 128)
  // and K = the padded rows (q_col_kchunks = A_pad_max / 128)
  int quant;
  uint8_t* q_sr; uint8_t* q_sc; int q_row_kchunks; int q_col_kchunks;
  int32_t* status;
};

struct Tile {
  int e, row0, m0, nt, nkb, krow0;
};

__device__ __forceinline__ int find_expert(const int* poff_s, int E, int row) {
  int lo = 0, hi = E - 1;       // largest e with poff[e] <= row
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (poff_s[mid] <= row) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// four consecutive entries of the gather map starting at padded row r (a
// multiple of 4): token rows, with pad rows mapped to the out-of-range row
__device__ __forceinline__ int4 gather_rows(const Params& p, int r) {
  int4 v = __ldg(reinterpret_cast<const int4*>(p.a_src + r));
  v.x = v.x < 0 ? p.a_oob : v.x;
  v.y = v.y < 0 ? p.a_oob : v.y;
  v.z = v.z < 0 ? p.a_oob : v.z;
  v.w = v.w < 0 ? p.a_oob : v.w;
  return v;
}

__device__ __forceinline__ Tile decode(const Params& p, const int* poff_s, int tile) {
  Tile t;
  if (!p.wgrad) {
    const int mt = tile / p.n_tiles;
    t.nt = tile - mt * p.n_tiles;
    t.row0 = mt * BM;
    t.e = p.dense_rows ? 0 : find_expert(poff_s, p.E, t.row0);
    t.m0 = t.row0;
    t.nkb = p.num_kb;
    t.krow0 = 0;
  } else {
    const int per_e = p.m_tiles_w * p.n_tiles;
    t.e = tile / per_e;
    const int rem = tile - t.e * per_e;
    const int mt = rem / p.n_tiles;
    t.nt = rem - mt * p.n_tiles;
    t.m0 = mt * BM;
    t.row0 = 0;
    t.krow0 = poff_s[t.e];
    t.nkb = -1;   // set by the caller from the group size and BK
  }
  return t;
}

__device__ __forceinline__ uint32_t bf16x2_bits(float a, float b) { return pack2(a, b); }

// barrier over a subset of the CTA's warps (id 0 is __syncthreads')
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// silu(z) = z sigmoid(z); the quotient is the 2-ulp fast division (the
// correctly rounded one costs more than the rest of the epilogue)
__device__ __forceinline__ float silu_f(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

template <bool MX>
__device__ __forceinline__ constexpr uint32_t make_idesc(bool a_mn, bool b_mn) {
  if constexpr (!MX) {
    return (1u << 4)              // D: fp32
           | (1u << 7)            // A: bf16
           | (1u << 10)           // B: bf16
           | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
  } else {
    return (0u << 7) | (0u << 10)   // A, B: E4M3
           | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(BN >> 3) << 17) | (1u << 23)   // scales: E8M0
           | ((uint32_t)(BM >> 4) << 24);
  }
}

template <bool MX, bool A_MN, int BLOAD, int EPI, bool GATHER = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmB3,
                    const __grid_constant__ CUtensorMap tmC,
                    const __grid_constant__ CUtensorMap tmC2,
                    const __grid_constant__ CUtensorMap tmIn,
                    const __grid_constant__ CUtensorMap tmQr,
                    const __grid_constant__ CUtensorMap tmQc, const Params p) {
  using Cfg = EpiCfg<MX, EPI, A_MN>;      // A MN-major <=> weight-gradient tiles
  constexpr int STAGES = Cfg::STAGES;
  constexpr int STG = Cfg::STG;
  constexpr int B_STAGE = Cfg::B_STAGE;
  constexpr int SPLIT_BYTES = 128 * 128;   // router: one split's B tile (2 boxes)
  constexpr int ELEM = MX ? 1 : 2;
  constexpr int BK = 128 / ELEM;                 // K per stage (128-byte rows)
  constexpr int MMA_K = MX ? 32 : 16;
  constexpr int KSTEPS = BK / MMA_K;             // 4
  constexpr bool B_MNMAJOR = (BLOAD == B_MN || BLOAD == B_MN_DUAL_N);
  constexpr int MN_CHUNK = 128 / ELEM;           // MN elements per 128-byte swizzle row
  constexpr int MN_CHUNK_BYTES = BK * 128;       // one box of an MN-major operand
  constexpr int ACC_BUFS = MX ? 1 : 2;
  constexpr int SF_COL0 = 256 * ACC_BUFS;        // TMEM column of the first scale stage
  constexpr uint32_t TMEM_COLS = MX ? 512 : 512;
  // MXFP8 SwiGLU backward: bf16 copy of the accumulator (128 columns)
  constexpr int PARK_COL = 384;
  static_assert(!MX || SF_COL0 + 12 * Cfg::STAGES <= PARK_COL, "parked dh overlaps the scales");
  constexpr uint32_t STAGE_TX = A_BYTES + B_BYTES + (MX ? SFA_BYTES + SFB_BYTES : 0);

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES], empty_bar[STAGES];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], drain_bar;
  __shared__ __align__(8) uint64_t in_bar[NUM_EPI_WARPS][2];
  __shared__ uint32_t tmem_slot;
  __shared__ int poff_s[MAX_E + 1];
  __shared__ int krows_s[A_MN ? MAX_E : 1];  // wgrad: reduction rows of each group
  __shared__ volatile int abort_flag;
  __shared__ int gtok_s[GATHER ? BM : 1];    // gathered A: token of each row being copied
  __shared__ __align__(16) float qinv_s[MX ? NUM_EPI_WARPS : 1][32];   // quantising epilogues

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;                                  // STAGES x A_BYTES
  uint8_t* sB = smem + STAGES * A_BYTES;               // STAGES x B_STAGE
  uint8_t* sSF = sB + STAGES * B_STAGE;                // STAGES x (SFA + SFB), MX only
  uint8_t* sStg = sSF + (MX ? STAGES * (SFA_BYTES + SFB_BYTES) : 0);   // per-warp staging

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (!p.dense_rows)
    for (int i = threadIdx.x; i <= p.E; i += NUM_THREADS) poff_s[i] = p.poff[i];
  if constexpr (A_MN) {
    // a group's K loop stops after its last real row: padding rows are zero,
    // so whole K blocks of padding are not loaded and the last block issues
    // only the MMA K steps that hold real rows (the padded count otherwise)
    for (int e = threadIdx.x; e < p.E; e += NUM_THREADS)
      krows_s[e] = p.offsets ? p.offsets[e + 1] - p.offsets[e] : p.poff[e + 1] - p.poff[e];
  }
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      // gathered A: the B bytes' arrival plus one per producer lane's copies
      mbar_init(&full_bar[s], GATHER ? 1 + 32 : 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], NUM_EPI_WARPS);
    }
    mbar_init(&drain_bar, 1);
    for (int w = 0; w < NUM_EPI_WARPS; ++w) {
      mbar_init(&in_bar[w][0], 1);
      mbar_init(&in_bar[w][1], 1);
    }
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch(&tmA);
    tma_prefetch(&tmB);
    if (BLOAD == B_MN_DUAL_N || BLOAD == B_K_DUAL_K) tma_prefetch(&tmB3);
    tma_prefetch(&tmC);
    if (EPI == EPI_SWIGLU || (EPI == EPI_STORE && p.wgrad)) tma_prefetch(&tmC2);
    if (EPI == EPI_SWIGLU_BWD) tma_prefetch(&tmIn);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;

  const int total = p.wgrad ? p.E * p.m_tiles_w * p.n_tiles
                  : p.dense_rows ? ((p.dense_rows + BM - 1) / BM) * p.n_tiles
                                 : (poff_s[p.E] / BM) * p.n_tiles;
  auto group_kb = [&](const Tile& t) {
    if constexpr (A_MN) return (krows_s[t.e] + BK - 1) / BK;
    else return t.nkb;
  };

  if (warp == 0 && GATHER) {
    // ------------------------------------------------- producer (gathered A)
    // The whole warp copies the A rows from the unpermuted x with 16-byte
    // cp.async (completion: each lane's cp.async.mbarrier.arrive.noinc on
    // the stage's full barrier, whose count includes the 32 lanes); lane 0
    // posts the B bytes and issues the B loads with TMA.  16-byte unit j of a
    // 128-byte shared-memory row r sits at (j ^ (r & 7)) * 16: the layout of
    // the TMA 128-byte swizzle the MMA descriptors expect.  A token row < 0
    // (a pad row) is zero-filled.
    //  rows mode: the tile's 128 rows x 64 K; lane l copies unit l % 8 of
    //    rows 4 i + l / 8, i = 0..31;
    //  weight-gradient mode: the stage's 64 K rows (tokens) x the tile's 128
    //    M columns, two 64-column chunks; lane l copies unit l % 8 of rows
    //    4 i + l / 8 of both chunks, i = 0..15.
    int stage = 0;
    uint32_t phase = 0;
    uint32_t used = 0, last_parity = 0;
    bool stop = false;
    const __nv_bfloat16* xb = p.a_x;
    const int j = lane & 7;
    for (int tile = blockIdx.x; tile < total && !stop; tile += gridDim.x) {
      const Tile t = decode(p, poff_s, tile);
      const int nkb = group_kb(t);
      if constexpr (!A_MN) {
        const int4 v = __ldg(reinterpret_cast<const int4*>(p.a_src + t.row0 + 4 * lane));
        __syncwarp();
        gtok_s[4 * lane] = v.x; gtok_s[4 * lane + 1] = v.y;
        gtok_s[4 * lane + 2] = v.z; gtok_s[4 * lane + 3] = v.w;
        __syncwarp();
      }
      for (int kb = 0; kb < nkb; ++kb) {
        int ok = 1;
        if (lane == 0)
          ok = mbar_wait(&empty_bar[stage], phase ^ 1, &abort_flag, p.status, kWaitLimitNs);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) { stop = true; break; }
        uint64_t* fb = &full_bar[stage];
        if constexpr (A_MN) {
          __syncwarp();
          if (lane < 16) {
            const int4 v = __ldg(reinterpret_cast<const int4*>(p.a_src + t.krow0 + kb * BK + 4 * lane));
            gtok_s[4 * lane] = v.x; gtok_s[4 * lane + 1] = v.y;
            gtok_s[4 * lane + 2] = v.z; gtok_s[4 * lane + 3] = v.w;
          }
          __syncwarp();
        }
        if (lane == 0) mbar_arrive_expect_tx(fb, STAGE_TX - A_BYTES);
        uint8_t* a_dst = sA + stage * A_BYTES;
        if constexpr (!A_MN) {
#pragma unroll 8
          for (int i = 0; i < 32; ++i) {
            const int r = 4 * i + (lane >> 3);
            const int tk = gtok_s[r];
            const __nv_bfloat16* src = tk >= 0 ? xb + (size_t)tk * p.a_ld + kb * BK + j * 8 : xb;
            cp_async16(a_dst + r * 128 + ((j ^ (r & 7)) << 4), src, tk >= 0);
          }
        } else {
#pragma unroll 8
          for (int i = 0; i < 16; ++i) {
            const int r = 4 * i + (lane >> 3);
            const int tk = gtok_s[r];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const __nv_bfloat16* src =
                  tk >= 0 ? xb + (size_t)tk * p.a_ld + t.m0 + c * MN_CHUNK + j * 8 : xb;
              cp_async16(a_dst + c * MN_CHUNK_BYTES + r * 128 + ((j ^ (r & 7)) << 4), src, tk >= 0);
            }
          }
        }
        cp_async_arrive_noinc(fb);
        if (lane == 0) {
          uint8_t* b_dst = sB + stage * B_STAGE;
          const int brow = p.wgrad ? t.krow0 : t.e * p.b_rows_per_e;
          if constexpr (BLOAD == B_MN) {
            tma_load_3d(b_dst, &tmB, fb, 0, brow + kb * BK, t.nt * BN / MN_CHUNK);
          } else if constexpr (BLOAD == B_MN_DUAL_N) {
            constexpr int HALF_CHUNKS = (BN / 2) / MN_CHUNK;
            tma_load_3d(b_dst, &tmB, fb, 0, brow + kb * BK, t.nt * (BN / 2) / MN_CHUNK);
            tma_load_3d(b_dst + HALF_CHUNKS * MN_CHUNK_BYTES, &tmB3, fb, 0, brow + kb * BK,
                        t.nt * (BN / 2) / MN_CHUNK);
          }
        }
        used |= 1u << stage;
        last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
    if (lane == 0)     // every copy and load of the warp has landed before the CTA exits
      for (int s = 0; s < STAGES; ++s)
        if (used & (1u << s)) {
          volatile int no_abort = 0;
          mbar_wait(&full_bar[s], (last_parity >> s) & 1, &no_abort, p.status, kWaitLimitNs);
        }
  } else if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t used = 0;               // stages that ever received a load
      uint32_t last_parity = 0;        // parity of the last load per stage (bit s)
      for (int tile = blockIdx.x; tile < total && !abort_flag; tile += gridDim.x) {
        const Tile t = decode(p, poff_s, tile);
        const int nkb = group_kb(t);
        for (int step = 0; step < nkb; ++step) {
          // the router's tiles all read the same split weights: each tile
          // starts at its own K block so that they do not stream the same
          // lines at the same time (fp32 sums in a rotated, fixed order)
          const int kb = is_router(EPI) ? (step + tile) % nkb : step;
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_flag, p.status, kWaitLimitNs)) break;
          uint64_t* fb = &full_bar[stage];
          const int nbox = p.b_boxes ? p.b_boxes : BN / MN_CHUNK;
          if constexpr (is_router(EPI))
            mbar_arrive_expect_tx(fb, A_BYTES + 2 * nbox * MN_CHUNK_BYTES);
          else
            mbar_arrive_expect_tx(fb, B_MNMAJOR ? STAGE_TX - (BN / MN_CHUNK - nbox) * MN_CHUNK_BYTES
                                                : STAGE_TX);
          uint8_t* a_dst = sA + stage * A_BYTES;
          uint8_t* b_dst = sB + stage * B_STAGE;
          // A operand
          if constexpr (!A_MN) {
            tma_load_2d(a_dst, &tmA, fb, kb * BK, t.row0);
          } else if (p.a3d) {
            tma_load_3d(a_dst, &tmA, fb, 0, t.krow0 + kb * BK, t.m0 / MN_CHUNK);
          } else {
#pragma unroll
            for (int i = 0; i < BM / MN_CHUNK; ++i)
              tma_load_2d(a_dst + i * MN_CHUNK_BYTES, &tmA, fb, t.m0 + i * MN_CHUNK,
                          t.krow0 + kb * BK);
          }
          // B operand
          const int brow = p.wgrad ? t.krow0 : t.e * p.b_rows_per_e;
          if constexpr (is_router(EPI)) {
            // rows kb*BK.. of each weight split (split s starts at row s * d)
            for (int sp = 0; sp < 2; ++sp)
              for (int i = 0; i < nbox; ++i)
                tma_load_2d(b_dst + sp * SPLIT_BYTES + i * MN_CHUNK_BYTES, &tmB, fb, i * MN_CHUNK,
                            sp * p.split_rows + kb * BK);
          } else if constexpr (BLOAD == B_MN) {
            if (p.b3d) {
              tma_load_3d(b_dst, &tmB, fb, 0, brow + kb * BK, t.nt * BN / MN_CHUNK);
            } else {
#pragma unroll
              for (int i = 0; i < nbox; ++i)
                tma_load_2d(b_dst + i * MN_CHUNK_BYTES, &tmB, fb, t.nt * BN + i * MN_CHUNK,
                            brow + kb * BK);
            }
          } else if constexpr (BLOAD == B_MN_DUAL_N) {
            constexpr int HALF_CHUNKS = (BN / 2) / MN_CHUNK;
            if (p.b3d) {
              tma_load_3d(b_dst, &tmB, fb, 0, brow + kb * BK, t.nt * (BN / 2) / MN_CHUNK);
              tma_load_3d(b_dst + HALF_CHUNKS * MN_CHUNK_BYTES, &tmB3, fb, 0, brow + kb * BK,
                          t.nt * (BN / 2) / MN_CHUNK);
            } else
#pragma unroll
            for (int i = 0; i < HALF_CHUNKS; ++i) {
              tma_load_2d(b_dst + i * MN_CHUNK_BYTES, &tmB, fb, t.nt * (BN / 2) + i * MN_CHUNK,
                          brow + kb * BK);
              tma_load_2d(b_dst + (HALF_CHUNKS + i) * MN_CHUNK_BYTES, &tmB3, fb,
                          t.nt * (BN / 2) + i * MN_CHUNK, brow + kb * BK);
            }
          } else if constexpr (BLOAD == B_K) {
            tma_load_2d(b_dst, &tmB, fb, kb * BK, brow + t.nt * BN);
          } else {
            const int k = kb * BK;
            if (k < p.k_split) tma_load_2d(b_dst, &tmB, fb, k, brow + t.nt * BN);
            else tma_load_2d(b_dst, &tmB3, fb, k - p.k_split, brow + t.nt * BN);
          }
          if constexpr (MX) {
            uint8_t* sf = sSF + stage * (SFA_BYTES + SFB_BYTES);
            // A scales: one 512-byte chunk (128 MN rows x 4 K blocks)
            long long ca;
            if constexpr (!A_MN) ca = (long long)(t.row0 / 128) * p.a_sc_kchunks + kb;
            else ca = (long long)(t.m0 / 128) * p.a_sc_kchunks + (t.krow0 / 128 + kb);
            bulk_load(sf, p.a_sc + ca * 512, SFA_BYTES, fb);
            // B scales: two chunks (N rows 0..127 and 128..255 of the tile)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint8_t* base = p.b_sc;
              long long cb;
              if constexpr (BLOAD == B_MN) {
                const long long nb = (long long)(t.nt * BN) / 128 + h;
                cb = nb * p.b_sc_kchunks + (brow / 128 + kb);
              } else if constexpr (BLOAD == B_MN_DUAL_N) {
                base = h ? p.b3_sc : p.b_sc;
                cb = (long long)t.nt * p.b_sc_kchunks + (brow / 128 + kb);
              } else if constexpr (BLOAD == B_K) {
                cb = ((long long)(brow + t.nt * BN) / 128 + h) * p.b_sc_kchunks + kb;
              } else {
                const int k = kb * BK;
                int kk = kb;
                if (k >= p.k_split) { base = p.b3_sc; kk = (k - p.k_split) / BK; }
                cb = ((long long)(brow + t.nt * BN) / 128 + h) * p.b_sc_kchunks + kk;
              }
              bulk_load(sf + SFA_BYTES + h * 512, base + cb * 512, 512, fb);
            }
          }
          used |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // drain: every load this thread issued has landed before the CTA exits
      for (int s = 0; s < STAGES; ++s)
        if (used & (1u << s)) {
          volatile int no_abort = 0;
          mbar_wait(&full_bar[s], (last_parity >> s) & 1, &no_abort, p.status, kWaitLimitNs);
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t IDESC = make_idesc<MX>(A_MN, B_MNMAJOR);
      const uint32_t idesc =
          p.mma_n ? (IDESC & ~(0x3Fu << 17)) | ((uint32_t)(p.mma_n >> 3) << 17) : IDESC;
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
      for (int tile = blockIdx.x; tile < total && !abort_flag; tile += gridDim.x, ++it) {
        const Tile t = decode(p, poff_s, tile);
        const int nkb = group_kb(t);
        const int acc = ACC_BUFS == 2 ? (it & 1) : 0;
        const uint32_t acc_par = ACC_BUFS == 2 ? ((it >> 1) & 1) : (it & 1);
        if (!mbar_wait(&acc_empty[acc], acc_par ^ 1, &abort_flag, p.status, kWaitLimitNs)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * 256;
        // K steps of the group's last block that hold real rows (wgrad)
        int last_ks = KSTEPS;
        if constexpr (A_MN) last_ks = (krows_s[t.e] - (nkb - 1) * BK + MMA_K - 1) / MMA_K;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, &abort_flag, p.status, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // gathered A was written by cp.async (generic proxy): order it
          // before the tensor core's reads (async proxy)
          if constexpr (GATHER) fence_async_smem();
          const uint32_t sa = a_base + stage * A_BYTES, sb = b_base + stage * B_STAGE;
          uint32_t sfa_t = 0, sfb_t = 0;
          if constexpr (MX) {
            const uint32_t sf = smem_u32(sSF + stage * (SFA_BYTES + SFB_BYTES));
            sfa_t = tmem_base + SF_COL0 + stage * 12;
            sfb_t = sfa_t + 4;
            tmem_cp_32x128b_warpx4(sfa_t, smem_desc(sf, 0, 128, 0));
            tmem_cp_32x128b_warpx4(sfb_t, smem_desc(sf + SFA_BYTES, 0, 128, 0));
            tmem_cp_32x128b_warpx4(sfb_t + 4, smem_desc(sf + SFA_BYTES + 512, 0, 128, 0));
          }
          if constexpr (is_router(EPI)) {
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ++ks) {
              const uint64_t ad = smem_desc(sa + ks * 32, 16, 1024, 2);
#pragma unroll
              for (int sp = 0; sp < 2; ++sp) {
                const uint64_t bd =
                    smem_desc(sb + sp * SPLIT_BYTES + ks * MMA_K * 128, MN_CHUNK_BYTES, 1024, 2);
                mma_bf16(d_tmem, ad, bd, idesc, (kb > 0 || ks > 0 || sp > 0) ? 1u : 0u);
              }
            }
          } else
#pragma unroll
          for (int ks = 0; ks < KSTEPS; ++ks) {
            if (A_MN && kb == nkb - 1 && ks >= last_ks) break;
            uint64_t ad, bd;
            if constexpr (!A_MN) ad = smem_desc(sa + ks * 32, 16, 1024, 2);
            else ad = smem_desc(sa + ks * MMA_K * 128, MN_CHUNK_BYTES, 1024, 2);
            if constexpr (!B_MNMAJOR) bd = smem_desc(sb + ks * 32, 16, 1024, 2);
            else bd = smem_desc(sb + ks * MMA_K * 128, MN_CHUNK_BYTES, 1024, 2);
            const uint32_t accum = (kb > 0 || ks > 0) ? 1u : 0u;
            if constexpr (!MX) {
              mma_bf16(d_tmem, ad, bd, idesc, accum);
            } else {
              const uint32_t id = idesc | ((uint32_t)ks << 4) | ((uint32_t)ks << 29);
              mma_mxf8(d_tmem, ad, bd, id, accum, sfa_t, sfb_t);
            }
          }
          mma_commit(&empty_bar[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (nkb > 0) mma_commit(&acc_full[acc]);
        else mbar_arrive(&acc_full[acc]);      // empty group: the epilogue writes zeros
      }
      // drain: all issued MMAs have completed before TMEM is released
      mma_commit(&drain_bar);
      volatile int no_abort = 0;
      mbar_wait(&drain_bar, 0, &no_abort, p.status, kWaitLimitNs);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int ew = warp - 2;                // epilogue warp 0..7
    const int hc = ew >> 2;                 // which half of the tile's columns
    const int r = lane;                     // row inside the warp's 32-row box
    uint8_t* stg = sStg + ew * STG;         // this warp's staging boxes
    uint32_t in_phase = 0;                  // bit i: parity of in_bar[ew][i]
    uint32_t in_pending = 0;                // bit i: a load into pair i not yet waited for (lane 0)
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      const Tile t = decode(p, poff_s, tile);
      const int nkb = group_kb(t);
      const int acc = ACC_BUFS == 2 ? (it & 1) : 0;
      const uint32_t acc_par = ACC_BUFS == 2 ? ((it >> 1) & 1) : (it & 1);
      const bool empty = nkb <= 0;
      const int y0 = (p.wgrad ? t.e * p.k_out + t.m0 : t.row0) + q * 32;

      if constexpr (EPI == EPI_SWIGLU_BWD) {
        // H1/H3 chunk 0 does not depend on the accumulator: fetch it now
        if (lane == 0) {
          const int c0 = t.nt * BN + hc * (BN / 2);
          bulk_wait_read<0>();
          mbar_arrive_expect_tx(&in_bar[ew][0], 2 * BOX_BYTES);
          tma_load_2d(stg, &tmIn, &in_bar[ew][0], c0, y0);
          tma_load_2d(stg + BOX_BYTES, &tmIn, &in_bar[ew][0], p.half + c0, y0);
          in_pending |= 1u;
        }
      }
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&acc_full[acc], acc_par, &abort_flag, p.status, kWaitLimitNs);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * 256;

      // EARLY: this thread's accumulator slice goes to registers at once and
      // the accumulator is handed back to the MMA warp before any store is
      // made.  Used where TMEM holds a single accumulator (MXFP8) and the
      // epilogue keeps no other large state; otherwise each 32-column chunk
      // is read from TMEM when it is stored and the accumulator is released
      // at the end of the tile (BF16 double-buffers its accumulators).
      // (the SwiGLU backward keeps the per-chunk path: with its whole slice
      // in registers it spills, measured 2.3x slower)
      constexpr bool EARLY = MX && (EPI == EPI_STORE || EPI == EPI_SWIGLU);
      // PARK (MXFP8 SwiGLU backward, whose working set leaves no room for
      // the slice in registers): dh is the bf16 output of GEMM2's dgrad, so
      // the slice is rounded to bf16 pairs and parked in TMEM columns the
      // MMA does not use (PARK_COL + 64 hc + [0, 64), past the accumulator
      // and the scale stages); the accumulator is handed back at once and
      // each chunk reads its 16 packed columns from the parked copy
      constexpr bool PARK = MX && EPI == EPI_SWIGLU_BWD;
      constexpr int NV = EARLY ? 128 : 32;
      uint32_t av[NV];
      const uint32_t park = tmem_base + ((uint32_t)(q * 32) << 16) + PARK_COL + hc * 64;
      if constexpr (PARK) {
        if (!empty) {
#pragma unroll 1
          for (int i = 0; i < 4; ++i) {
            tmem_ld32(tbase + hc * (BN / 2) + 32 * i, av);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int m = 0; m < 16; ++m)
              pk[m] = bf16x2_bits(__uint_as_float(av[2 * m]), __uint_as_float(av[2 * m + 1]));
            tmem_st16(park + 16 * i, pk);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc]);
      }
      if constexpr (EARLY) {
        if (!empty) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            // STORE / SwiGLU-bwd: columns hc*128 + [0,128); SwiGLU: W1 part
            // hc*64 + [0,64) then W3 part 128 + hc*64 + [0,64)
            const uint32_t col = EPI == EPI_SWIGLU ? (i >> 1) * (BN / 2) + hc * 64 + (i & 1) * 32
                                                   : hc * (BN / 2) + i * 32;
            tmem_ld32(tbase + col, av + 32 * i);
          }
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < NV; ++i) av[i] = 0u;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc]);
      }

      if constexpr (EPI == EPI_STORE) {
        const int n0 = t.nt * BN;
        const CUtensorMap* map = &tmC;
        int x0 = n0;
        if (p.wgrad && p.n_split > 0 && n0 >= p.n_split) { map = &tmC2; x0 = n0 - p.n_split; }
        // rank-1 term (rows mode): this thread's row scale and the expert's column vector
        const bool r1 = !p.wgrad && p.row_scale != nullptr;
        const float rs = r1 ? p.row_scale[y0 + r] : 0.f;
        const float* cvec = r1 ? p.col_vec + (size_t)t.e * p.col_ld + n0 : nullptr;
#pragma unroll(EARLY ? 4 : 1)
        for (int ci = 0; ci < 4; ++ci) {
          const int c = hc * (BN / 2) + ci * CHUNK;
          const uint32_t* v = av + (EARLY ? 32 * ci : 0);
          if constexpr (!EARLY) {
            if (!empty) {
              tmem_ld32(tbase + c, av);
              tmem_wait_ld();
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) av[i] = 0u;
            }
          }
          constexpr int NB = Cfg::BOXES;
          uint8_t* buf = stg + (NB > 1 ? (ci & 1) * BOX_BYTES : 0);
          if (lane == 0) {                       // the store that last used `buf` has read it
            if constexpr (NB > 1) bulk_wait_read<1>();
            else bulk_wait_read<0>();
          }
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float f[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = __uint_as_float(v[8 * j + i]);
            if (r1) {
              const float4* cv = reinterpret_cast<const float4*>(cvec + c + 8 * j);
              const float4 c0 = __ldg(cv), c1 = __ldg(cv + 1);
              f[0] = fmaf(rs, c0.x, f[0]); f[1] = fmaf(rs, c0.y, f[1]);
              f[2] = fmaf(rs, c0.z, f[2]); f[3] = fmaf(rs, c0.w, f[3]);
              f[4] = fmaf(rs, c1.x, f[4]); f[5] = fmaf(rs, c1.y, f[5]);
              f[6] = fmaf(rs, c1.z, f[6]); f[7] = fmaf(rs, c1.w, f[7]);
            }
            uint4 w;
            w.x = bf16x2_bits(f[0], f[1]);
            w.y = bf16x2_bits(f[2], f[3]);
            w.z = bf16x2_bits(f[4], f[5]);
            w.w = bf16x2_bits(f[6], f[7]);
            *reinterpret_cast<uint4*>(buf + sw64(r, j)) = w;
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(map, buf, x0 + c, y0);
            bulk_commit();
          }
        }
      } else if constexpr (EPI == EPI_SWIGLU) {
        // accumulator columns [0,128) = A W1, [128,256) = A W3 for the output
        // columns [nt*128, nt*128 + 128)
        const int n0 = t.nt * (BN / 2);
#pragma unroll(EARLY ? 2 : 1)
        for (int ci = 0; ci < 2; ++ci) {
          const int c = hc * (BN / 4) + ci * CHUNK;
          uint32_t gl[EARLY ? 1 : 32], ul[EARLY ? 1 : 32];
          if constexpr (!EARLY) {
            tmem_ld32(tbase + c, gl);
            tmem_ld32(tbase + BN / 2 + c, ul);
            tmem_wait_ld();
          }
          const uint32_t* g = EARLY ? av + 32 * ci : gl;        // A W1
          const uint32_t* u = EARLY ? av + 64 + 32 * ci : ul;   // A W3
          constexpr bool ONE_BOX = Cfg::BOXES == 1;
          if (lane == 0) bulk_wait_read<0>();
          __syncwarp();
          uint4 hkeep[ONE_BOX ? 4 : 1], gkeep[ONE_BOX ? 4 : 1], ukeep[ONE_BOX ? 4 : 1];
          const bool q = MX && p.quant;       // h leaves as MX codes, not bf16
          uint32_t hbits[MX ? 16 : 1];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4 hw, gw, uw;
            uint32_t* hp = &hw.x;
            uint32_t* gp = &gw.x;
            uint32_t* up = &uw.x;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float g0 = __uint_as_float(g[8 * j + 2 * i]);
              const float g1 = __uint_as_float(g[8 * j + 2 * i + 1]);
              const float u0 = __uint_as_float(u[8 * j + 2 * i]);
              const float u1 = __uint_as_float(u[8 * j + 2 * i + 1]);
              hp[i] = bf16x2_bits(silu_f(g0) * u0, silu_f(g1) * u1);
              gp[i] = bf16x2_bits(g0, g1);
              up[i] = bf16x2_bits(u0, u1);
            }
            if constexpr (ONE_BOX) {
              hkeep[j] = hw; gkeep[j] = gw; ukeep[j] = uw;
            } else {
              if constexpr (MX) {
                hbits[4 * j] = hw.x; hbits[4 * j + 1] = hw.y;
                hbits[4 * j + 2] = hw.z; hbits[4 * j + 3] = hw.w;
              }
              if (!q) *reinterpret_cast<uint4*>(stg + sw64(r, j)) = hw;
              *reinterpret_cast<uint4*>(stg + BOX_BYTES + sw64(r, j)) = gw;
              *reinterpret_cast<uint4*>(stg + 2 * BOX_BYTES + sw64(r, j)) = uw;
            }
          }
          if constexpr (MX && !ONE_BOX) {
            if (q) {
              // the bf16-rounded h of this warp's 32 x 32 block, quantised
              // along F (fwd GEMM2) and down the rows (GEMM2 weight grad)
              float hv[32];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hbits[i]));
                hv[2 * i] = f2.x;
                hv[2 * i + 1] = f2.y;
              }
              mx_quant_block32(hv, hbits, stg, stg + 1024, p.q_sr, y0 + r, n0 + c, p.q_row_kchunks,
                               p.q_sc, y0, p.q_col_kchunks, qinv_s[MX ? ew : 0]);
            }
          }
          if constexpr (ONE_BOX) {
            // one staging box: h, then H1, then H3, each stored before the next
            const uint4* outs[3] = {hkeep, gkeep, ukeep};
#pragma unroll
            for (int o = 0; o < 3; ++o) {
              if (o > 0 && !p.aux) break;
              if (o > 0) {
                if (lane == 0) bulk_wait_read<0>();
                __syncwarp();
              }
#pragma unroll
              for (int j = 0; j < 4; ++j) *reinterpret_cast<uint4*>(stg + sw64(r, j)) = outs[o][j];
              fence_async_smem();
              __syncwarp();
              if (lane == 0) {
                if (o == 0) tma_store_2d(&tmC, stg, n0 + c, y0);
                else tma_store_2d(&tmC2, stg, (o == 2 ? p.half : 0) + n0 + c, y0);
                bulk_commit();
              }
            }
          } else {
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (q) {
                tma_store_2d(&tmQr, stg, n0 + c, y0);
                tma_store_2d(&tmQc, stg + 1024, n0 + c, y0);
              } else {
                tma_store_2d(&tmC, stg, n0 + c, y0);
              }
              if (p.aux) {
                tma_store_2d(&tmC2, stg + BOX_BYTES, n0 + c, y0);
                tma_store_2d(&tmC2, stg + 2 * BOX_BYTES, p.half + n0 + c, y0);
              }
              bulk_commit();
            }
          }
        }
      } else if constexpr (EPI == EPI_SWIGLU_BWD) {  // accumulator = dh, columns [nt*256, +256)
        const int n0 = t.nt * BN + hc * (BN / 2);
        constexpr int NCH = BN / 2 / CHUNK;
#pragma unroll 1
        for (int ci = 0; ci < NCH; ++ci) {
          const int c = ci * CHUNK;
          const int pr = ci & 1;                      // staging pair of this chunk
          uint8_t* b1 = stg + pr * 2 * BOX_BYTES;
          uint8_t* b3 = b1 + BOX_BYTES;
          if (ci + 1 < NCH && lane == 0) {            // prefetch the next chunk's H1/H3
            uint8_t* n1 = stg + (pr ^ 1) * 2 * BOX_BYTES;
            bulk_wait_read<0>();                      // its pair's previous stores have read it
            mbar_arrive_expect_tx(&in_bar[ew][pr ^ 1], 2 * BOX_BYTES);
            tma_load_2d(n1, &tmIn, &in_bar[ew][pr ^ 1], n0 + c + CHUNK, y0);
            tma_load_2d(n1 + BOX_BYTES, &tmIn, &in_bar[ew][pr ^ 1], p.half + n0 + c + CHUNK, y0);
            in_pending |= 1u << (pr ^ 1);
          }
          uint32_t* v = av;
          if constexpr (PARK) {
            // this chunk's dh: 16 parked bf16 pairs -> 32 fp32 bit patterns
            uint32_t pk[16];
            if (!empty) {
              tmem_ld16(park + 16 * ci, pk);
              tmem_wait_ld();
            } else {
#pragma unroll
              for (int m = 0; m < 16; ++m) pk[m] = 0u;
            }
#pragma unroll
            for (int m = 0; m < 16; ++m) {
              v[2 * m] = pk[m] << 16;
              v[2 * m + 1] = pk[m] & 0xffff0000u;
            }
          } else {
            tmem_ld32(tbase + hc * (BN / 2) + c, v);
            tmem_wait_ld();
          }
          int got = 1;
          if (lane == 0)
            got = mbar_wait(&in_bar[ew][pr], (in_phase >> pr) & 1, &abort_flag, p.status,
                            kWaitLimitNs);
          got = __shfl_sync(0xffffffffu, got, 0);
          if (got) {
            in_phase ^= 1u << pr;
            in_pending &= ~(1u << pr);
          }
          if (!got) { ok = 0; break; }
          const bool q = MX && p.quant;     // dA1 | dA3 leave as MX codes, not bf16
          uint4 o1k[MX ? 4 : 1], o3k[MX ? 4 : 1];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float f1[8], f3[8], o1[8], o3[8];
            unpack8(*reinterpret_cast<const uint4*>(b1 + sw64(r, j)), f1);
            unpack8(*reinterpret_cast<const uint4*>(b3 + sw64(r, j)), f3);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float dh = __uint_as_float(v[8 * j + i]);
              const float z = f1[i];
              const float sg = __fdividef(1.0f, 1.0f + __expf(-z));
              o1[i] = dh * f3[i] * sg * (1.0f + z * (1.0f - sg));
              o3[i] = dh * z * sg;
            }
            const uint4 w1 = pack8(o1), w3 = pack8(o3);
            if constexpr (MX) {
              o1k[j] = w1;
              o3k[j] = w3;
            }
            if (!q) {
              *reinterpret_cast<uint4*>(b1 + sw64(r, j)) = w1;
              *reinterpret_cast<uint4*>(b3 + sw64(r, j)) = w3;
            }
          }
          if constexpr (MX) {
            if (q) {
              // the bf16-rounded dA1 and dA3 of this warp's 32 x 32 blocks,
              // quantised along 2F (GEMM1 dgrad) and down the rows (GEMM1
              // weight grad); the codes reuse the H1 / H3 boxes once every
              // lane has read its row of them
              __syncwarp();
#pragma unroll
              for (int o = 0; o < 2; ++o) {
                const uint4* k4 = o == 0 ? o1k : o3k;
                float dv[32];
#pragma unroll
                for (int j = 0; j < 4; ++j) unpack8(k4[j], dv + 8 * j);
                uint8_t* box = o == 0 ? b1 : b3;
                mx_quant_block32(dv, reinterpret_cast<const uint32_t*>(k4), box, box + 1024, p.q_sr, y0 + r, (o ? p.half : 0) + n0 + c,
                                 p.q_row_kchunks, p.q_sc, y0, p.q_col_kchunks, qinv_s[MX ? ew : 0]);
              }
            }
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (q) {
              tma_store_2d(&tmQr, b1, n0 + c, y0);
              tma_store_2d(&tmQc, b1 + 1024, n0 + c, y0);
              tma_store_2d(&tmQr, b3, p.half + n0 + c, y0);
              tma_store_2d(&tmQc, b3 + 1024, p.half + n0 + c, y0);
            } else {
              tma_store_2d(&tmC, b1, n0 + c, y0);
              tma_store_2d(&tmC, b3, p.half + n0 + c, y0);
            }
            bulk_commit();
          }
        }
        if (!ok) break;
      } else {  // router: accumulator = fp32 logits, 128 tokens x E experts
        // Both column halves of the epilogue warps scan half of the experts
        // each for the running top-k of their token; the second half's list
        // is merged into the first through shared memory.  Ranks inside the
        // tile: each of four warps counts 32 tokens in order, then a prefix
        // over the four warps' counts (same result as one pass in token order).
        constexpr int KT = EPI == EPI_ROUTER4 ? 4 : 8;          // k <= KT
        int* sel_s = reinterpret_cast<int*>(sStg);              // [128][k] chosen experts
        float* mv_s = reinterpret_cast<float*>(sel_s + BM * KT);  // [128][k] second half's list
        int* me_s = reinterpret_cast<int*>(mv_s + BM * KT);
        int* rank_s = reinterpret_cast<int*>(mv_s);            // after the merge: in-warp ranks
        int* cnt4 = me_s;                                       // after the merge: [4][E] counts
        const int rloc = q * 32 + lane;
        const int row = t.row0 + rloc;
        const bool valid = row < p.dense_rows;
        const int k = p.r_k, E = p.r_E;
        const int ep = threadIdx.x - 64;                        // 0..255 over the epilogue warps
        const int lo = hc ? E / 2 : 0, hi = hc ? E : E / 2;
        float bv[KT];
        int be[KT];
#pragma unroll
        for (int i = 0; i < KT; ++i) { bv[i] = -INFINITY; be[i] = 0x7fffffff; }
#pragma unroll 1
        for (int c = lo; c < hi; c += 32) {
          uint32_t v[32];
          tmem_ld32(tbase + c, v);
          tmem_wait_ld();
          float L[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            L[i] = __uint_as_float(v[i]) + ((p.r_bias && c + i < hi) ? __ldg(p.r_bias + c + i) : 0.f);
          if (valid && p.r_logits) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              if (c + i < hi)
                *reinterpret_cast<float4*>(p.r_logits + (size_t)row * E + c + i) =
                    make_float4(L[i], L[i + 1], L[i + 2], L[i + 3]);
          }
          // experts arrive in increasing order, so a strict '>' keeps the
          // lower index first among equal logits
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (c + i >= hi) break;
            float cv = L[i];
            int ce = c + i;
            if (cv != cv) { cv = -INFINITY; if (valid) report(p.status, MOE_DEV_NONFINITE); }
#pragma unroll
            for (int s2 = 0; s2 < KT; ++s2) {
              if (cv > bv[s2]) {
                const float tv = bv[s2]; bv[s2] = cv; cv = tv;
                const int te = be[s2]; be[s2] = ce; ce = te;
              }
            }
          }
        }
        if (hc == 1)
#pragma unroll
          for (int j = 0; j < KT; ++j)
            if (j < k) { mv_s[rloc * k + j] = bv[j]; me_s[rloc * k + j] = be[j]; }
        named_bar_sync(1, 256);
        if (hc == 0) {
          // the second half's experts all have higher indices: a strict '>'
          // keeps the first half's entry ahead on equal logits
#pragma unroll
          for (int j = 0; j < KT; ++j) {
            if (j >= k) break;
            float cv = mv_s[rloc * k + j];
            int ce = me_s[rloc * k + j];
#pragma unroll
            for (int s2 = 0; s2 < KT; ++s2) {
              if (cv > bv[s2]) {
                const float tv = bv[s2]; bv[s2] = cv; cv = tv;
                const int te = be[s2]; be[s2] = ce; ce = te;
              }
            }
          }
          float ssum = 0.f;
#pragma unroll
          for (int j = 0; j < KT; ++j)
            if (j < k) ssum += expf(bv[j] - bv[0]);
#pragma unroll
          for (int j = 0; j < KT; ++j) {
            if (j >= k) continue;
            if (valid) {
              p.r_topk[(size_t)row * k + j] = be[j];
              p.r_gates[(size_t)row * k + j] = expf(bv[j] - bv[0]) / ssum;
            }
            sel_s[rloc * k + j] = valid ? be[j] : -1;
          }
        }
        named_bar_sync(1, 256);                  // sel_s complete; the merge buffers are free
        for (int i = ep; i < 4 * E; i += 256) cnt4[i] = 0;
        named_bar_sync(1, 256);
        if (hc == 0) {
          // warp ew counts tokens [32 ew, 32 ew + 32) in order, lane j = slot j
          int* cw = cnt4 + ew * E;
          for (int tt = 0; tt < 32; ++tt) {
            const int tok = ew * 32 + tt;
            if (lane < k) {
              const int e = sel_s[tok * k + lane];
              int rk = -1;
              if (e >= 0) { rk = cw[e]; cw[e] = rk + 1; }
              rank_s[tok * k + lane] = rk;
            }
            __syncwarp();
          }
        }
        named_bar_sync(1, 256);
        for (int e = ep; e < E; e += 256) {      // exclusive prefix over the warps; histogram
          int run = 0;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int n = cnt4[w * E + e];
            cnt4[w * E + e] = run;
            run += n;
          }
          p.r_hist[(size_t)(t.row0 / BM) * E + e] = run;
        }
        named_bar_sync(1, 256);
        if (hc == 0 && valid) {
#pragma unroll
          for (int j = 0; j < KT; ++j) {
            if (j >= k) continue;
            const int e = sel_s[rloc * k + j];
            int rk = rank_s[rloc * k + j];
            if (e >= 0) rk += cnt4[(rloc >> 5) * E + e];
            p.r_rank[(size_t)row * k + j] = rk;
          }
        }
        named_bar_sync(1, 256);                  // shared memory is reused by the next tile
      }
      if constexpr (!EARLY && !PARK) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc]);
      }
    }
    if (lane == 0) bulk_wait_all();     // every store has landed before the CTA exits
    if constexpr (EPI == EPI_SWIGLU_BWD) {
      // a prefetch issued for a tile that was then abandoned must land too
      if (lane == 0) {
        volatile int no_abort = 0;
        for (int i = 0; i < 2; ++i)
          if (in_pending & (1u << i))
            mbar_wait(&in_bar[ew][i], (in_phase >> i) & 1, &no_abort, p.status, kWaitLimitNs);
      }
    }
  }

  // every warp reconverges first: lanes that skipped a one-lane role loop
  // (producer, MMA issue) must not reach the CTA barrier, or the warp-wide
  // TMEM free after it, ahead of that lane
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side
// 2-D map over a row-major [outer, inner] array of 1- or 2-byte elements,
// box {box_inner, box_outer}, 128-byte swizzle.
moe_status_t make_map(CUtensorMap* m, const void* base, int elem_bytes, uint64_t inner,
                      uint64_t outer, uint32_t box_inner, uint32_t box_outer,
                      CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto fn = tensor_map_encoder();
  if (!fn) {
    set_error("cuTensorMapEncodeTiled unavailable");
    return MOE_ERR_CUDA;
  }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * (uint64_t)elem_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                  2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed (%d): inner %llu outer %llu box %u x %u", (int)r,
              (unsigned long long)inner, (unsigned long long)outer, box_inner, box_outer);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// 3-D view of a row-major [rows, cols] array as (chunk columns, rows, chunk
// index) with chunk = 128 bytes of a row: box (chunk, box_rows, nchunk) loads
// nchunk consecutive 128-byte column chunks of box_rows rows in one op, laid
// out in shared memory chunk after chunk (the MN-major operand layout).
// Returns false (map unusable) when the driver does not accept the view.
bool make_map_mn3(CUtensorMap* m, const void* base, int elem_bytes, uint64_t cols, uint64_t rows,
                  uint32_t box_rows, uint32_t nchunk) {
#ifdef MOE_GG_NO_3D
  return false;
#endif
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  const uint64_t ce = 128 / elem_bytes;
  if (cols % ce) return false;
  cuuint64_t dims[3] = {ce, rows, cols / ce};
  cuuint64_t strides[2] = {cols * (uint64_t)elem_bytes, 128};
  cuuint32_t box[3] = {(cuuint32_t)ce, box_rows, nchunk};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                  3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// epilogue box map: [outer, inner] bf16, 32 x 32 box, 64-byte swizzle
moe_status_t make_out_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer) {
  return make_map(m, base, 2, inner, outer, CHUNK, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

struct Maps {
  CUtensorMap a, b, b3, c, c2, in, qr, qc;
  bool q = false;     // qr / qc set (MX epilogue quantisation)
};

template <bool MX, bool A_MN, int BLOAD, int EPI, bool GATHER = false>
moe_status_t launch(const Maps& m, const Params& p, int max_tiles, cudaStream_t s) {
  auto kern = grouped_gemm_kernel<MX, A_MN, BLOAD, EPI, GATHER>;
  const size_t smem = EpiCfg<MX, EPI, A_MN>::SMEM;
  MOE_TRY(set_smem_limit(reinterpret_cast<const void*>(kern), smem, "grouped_gemm"));
  const int grid = max(1, min(num_sms(), max_tiles));
  kern<<<grid, NUM_THREADS, smem, s>>>(m.a, m.b, m.b3, m.c, m.c2, m.in, m.q ? m.qr : m.a,
                                       m.q ? m.qc : m.a, p);
  MOE_CHECK_LAUNCH("grouped_gemm");
  return MOE_OK;
}

}  // namespace gg
}  // namespace moe

using namespace moe;
using namespace moe::gg;

static Params base_params(const int32_t* poff, int E, int32_t* status) {
  Params p{};
  p.poff = poff;
  p.E = E;
  p.status = status;
  return p;
}

// Router logits on the tensor cores: x [T, d] (bf16) times W_r split exactly
// into two bf16 parts stacked as wsplit [2d, E] (w0 + w1 = W_r to within
// 2^-17 |W_r|): each stage holds one x tile and the two split tiles of the
// same K rows, and both products accumulate into one fp32 TMEM accumulator; top-k,
// gates, per-128-token-block ranks and histogram in the epilogue.
namespace moe {
moe_status_t router_tc(const void* x, const void* wsplit, const float* bias, int T, int d, int E,
                       int k, float* logits, int32_t* topk, float* gates, int32_t* rank,
                       int32_t* hist, int32_t* status, cudaStream_t s) {
  Params p = base_params(nullptr, 1, status);
  p.dense_rows = T;
  p.split_rows = d;        // split s of W_r starts at row s * d of wsplit
  p.num_kb = d / 64;
  p.b_rows_per_e = 0;
  p.n_tiles = 1;
  p.mma_n = (E + 15) / 16 * 16;
  p.b_boxes = (p.mma_n + 63) / 64;
  p.r_bias = bias;
  p.r_logits = logits;
  p.r_topk = topk;
  p.r_gates = gates;
  p.r_rank = rank;
  p.r_hist = hist;
  p.r_k = k;
  p.r_E = E;
  Maps m;
  MOE_TRY(make_map(&m.a, x, 2, d, T, 64, BM));
  MOE_TRY(make_map(&m.b, wsplit, 2, E, 2ULL * d, 64, 64));
  m.b3 = m.c = m.c2 = m.in = m.a;
  return k <= 4 ? launch<false, false, B_MN, EPI_ROUTER4>(m, p, (T + BM - 1) / BM, s)
                : launch<false, false, B_MN, EPI_ROUTER>(m, p, (T + BM - 1) / BM, s);
}
}  // namespace moe

// Self-test of the bounded pipeline wait: one thread waits on an mbarrier
// that nothing arrives at; after limit_ns the wait gives up, sets
// MOE_DEV_TIMEOUT in *status and the kernel returns.
namespace moe {
namespace gg {
__global__ void wait_timeout_selftest_kernel(int32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  mbar_init(&bar, 1);
  fence_barrier_init();
  mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
}
}  // namespace gg
}  // namespace moe

extern "C" moe_status_t moe_selftest_wait_timeout(int32_t* dev_status, uint64_t limit_ns,
                                                  moe_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  MOE_CHECK_ARG(dev_status != nullptr, "moe_selftest_wait_timeout: null status");
  MOE_CHECK_ARG(limit_ns > 0 && limit_ns <= 2000000000ull,
                "moe_selftest_wait_timeout: limit must be in (0, 2 s]");
  moe::gg::wait_timeout_selftest_kernel<<<1, 32, 0, s>>>(dev_status, limit_ns);
  MOE_CHECK_LAUNCH("wait_timeout_selftest");
  return MOE_OK;
}

// Forward grouped GEMM.  a_src == null: A is the permuted buffer
// [A_pad_max, K].  a_src != null (BF16): A is the unpermuted x [a_rows, K]
// and padded row r of the product reads x[a_src[r]] (a zero row where
// a_src[r] < 0), gathered by the producer with TMA row gathers.
static moe_status_t fwd_impl(int dt, const void* A, const uint8_t* A_sc, const void* B,
                             const uint8_t* B_sc, const void* B3, const uint8_t* B3_sc,
                             const int32_t* poff, int E, int A_pad_max, int N, int K,
                             int epilogue, void* C, void* aux, const int32_t* a_src, int a_rows,
                             int32_t* dev_status, cudaStream_t s) {
  const bool mx = dt == MOE_MXFP8;
  const bool gather = a_src != nullptr;
  MOE_CHECK_ARG(dt == MOE_BF16 || dt == MOE_MXFP8, "gemm_fwd: bad dtype");
  MOE_CHECK_ARG(!(gather && mx), "gemm_fwd: row gathers are BF16 only");
  MOE_CHECK_ARG(!gather || (a_rows > 0 && aligned16(a_src) && aligned16(A)),
                "gemm_fwd: gathered A needs T > 0 and 16-byte aligned x and src");
  MOE_CHECK_ARG(E > 0 && E <= MAX_E, "gemm_fwd: E must be in [1, %d]", MAX_E);
  MOE_CHECK_ARG(A_pad_max > 0 && A_pad_max % 128 == 0, "gemm_fwd: A_pad_max %% 128");
  MOE_CHECK_ARG(K > 0 && K % (mx ? 128 : 64) == 0, "gemm_fwd: K %% %d", mx ? 128 : 64);
  MOE_CHECK_ARG(A && B && C && poff, "gemm_fwd: null pointer");
  MOE_CHECK_ARG(!mx || (A_sc && B_sc), "gemm_fwd: MX needs scales");
  const int eb = mx ? 1 : 2;
  Params p = base_params(poff, E, dev_status);
  p.num_kb = K / (128 / eb);
  p.b_rows_per_e = K;
  p.a_sc = A_sc;
  p.a_sc_kchunks = K / 128;
  p.b_sc = B_sc;
  p.b3_sc = B3_sc;
  p.b_sc_kchunks = (int)((long long)E * K / 128);
  p.C = static_cast<__nv_bfloat16*>(C);
  p.a_src = a_src;
  p.a_oob = a_rows;
  p.a_x = static_cast<const __nv_bfloat16*>(A);
  p.a_ld = K;
  Maps m;
  if (gather) MOE_TRY(make_map(&m.a, A, 2, K, a_rows, 64, 1));   // unused by the gathering producer
  else MOE_TRY(make_map(&m.a, A, eb, K, A_pad_max, 128 / eb, BM));
  if (epilogue == MOE_EPI_NONE) {
    MOE_CHECK_ARG(N > 0 && N % 256 == 0, "gemm_fwd: N %% 256");
    p.n_tiles = N / BN;
    p.ldc = N;
    p.b3d = make_map_mn3(&m.b, B, eb, N, (uint64_t)E * K, 128 / eb, BN * eb / 128);
    if (!p.b3d) {
      MOE_CHECK_ARG(!gather, "gemm_fwd: gathered A needs the 3-D weight map");
      MOE_TRY(make_map(&m.b, B, eb, N, (uint64_t)E * K, 128 / eb, 128 / eb));
    }
    MOE_TRY(make_out_map(&m.c, C, N, A_pad_max));
    m.b3 = m.c2 = m.in = m.a;
    const int max_tiles = (A_pad_max / BM) * p.n_tiles;
    if (gather) return launch<false, false, B_MN, EPI_STORE, true>(m, p, max_tiles, s);
    return mx ? launch<true, false, B_MN, EPI_STORE>(m, p, max_tiles, s)
              : launch<false, false, B_MN, EPI_STORE>(m, p, max_tiles, s);
  }
  MOE_CHECK_ARG(epilogue == MOE_EPI_SWIGLU, "gemm_fwd: epilogue must be NONE or SWIGLU");
  MOE_CHECK_ARG(B3 && (!mx || B3_sc), "gemm_fwd: SWIGLU needs B3 (W3)");
  MOE_CHECK_ARG(N > 0 && N % 128 == 0, "gemm_fwd: SWIGLU needs F %% 128");
  p.n_tiles = N / (BN / 2);
  p.ldc = N;
  p.aux = static_cast<__nv_bfloat16*>(aux);
  p.ld_aux = 2LL * N;
  p.half = N;
  p.b3d = make_map_mn3(&m.b, B, eb, N, (uint64_t)E * K, 128 / eb, (BN / 2) * eb / 128) &&
          make_map_mn3(&m.b3, B3, eb, N, (uint64_t)E * K, 128 / eb, (BN / 2) * eb / 128);
  if (!p.b3d) {
    MOE_CHECK_ARG(!gather, "gemm_fwd: gathered A needs the 3-D weight maps");
    MOE_TRY(make_map(&m.b, B, eb, N, (uint64_t)E * K, 128 / eb, 128 / eb));
    MOE_TRY(make_map(&m.b3, B3, eb, N, (uint64_t)E * K, 128 / eb, 128 / eb));
  }
  MOE_TRY(make_out_map(&m.c, C, N, A_pad_max));
  if (aux) MOE_TRY(make_out_map(&m.c2, aux, 2ULL * N, A_pad_max));
  else m.c2 = m.c;
  m.in = m.a;
  const int max_tiles = (A_pad_max / BM) * p.n_tiles;
  if (gather) return launch<false, false, B_MN_DUAL_N, EPI_SWIGLU, true>(m, p, max_tiles, s);
  return mx ? launch<true, false, B_MN_DUAL_N, EPI_SWIGLU>(m, p, max_tiles, s)
            : launch<false, false, B_MN_DUAL_N, EPI_SWIGLU>(m, p, max_tiles, s);
}

extern "C" moe_status_t moe_grouped_gemm_fwd(int dt, const void* A, const uint8_t* A_sc,
                                             const void* B, const uint8_t* B_sc, const void* B3,
                                             const uint8_t* B3_sc, const int32_t* poff, int E,
                                             int A_pad_max, int N, int K, int epilogue, void* C,
                                             void* aux, int32_t* dev_status,
                                             moe_stream_t stream) {
  return fwd_impl(dt, A, A_sc, B, B_sc, B3, B3_sc, poff, E, A_pad_max, N, K, epilogue, C, aux,
                  nullptr, 0, dev_status, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" moe_status_t moe_grouped_gemm_fwd_gather(const void* x, int T, const int32_t* src,
                                                    const void* B, const void* B3,
                                                    const int32_t* poff, int E, int A_pad_max,
                                                    int N, int K, int epilogue, void* C,
                                                    void* aux, int32_t* dev_status,
                                                    moe_stream_t stream) {
  MOE_CHECK_ARG(x && src, "gemm_fwd_gather: null x or src");
  return fwd_impl(MOE_BF16, x, nullptr, B, nullptr, B3, nullptr, poff, E, A_pad_max, N, K,
                  epilogue, C, aux, src, T, dev_status, reinterpret_cast<cudaStream_t>(stream));
}

// MXFP8 forward GEMM1 with the SwiGLU epilogue whose h leaves as MX codes:
// along F (h_q / h_s, for the forward GEMM2) and down the rows (hT_q / hT_s,
// for the GEMM2 weight gradient), from the bf16-rounded h; aux [H1 | H3] as
// in moe_grouped_gemm_fwd.  h itself is not stored.
extern "C" moe_status_t moe_grouped_gemm_fwd_swiglu_mxq(
    const void* A, const uint8_t* A_sc, const void* B, const uint8_t* B_sc, const void* B3,
    const uint8_t* B3_sc, const int32_t* poff, int E, int A_pad_max, int F, int K, void* aux,
    uint8_t* h_q, uint8_t* h_s, uint8_t* hT_q, uint8_t* hT_s, int32_t* dev_status,
    moe_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  MOE_CHECK_ARG(E > 0 && E <= MAX_E, "gemm_fwd_swiglu_mxq: E must be in [1, %d]", MAX_E);
  MOE_CHECK_ARG(A_pad_max > 0 && A_pad_max % 128 == 0, "gemm_fwd_swiglu_mxq: A_pad_max %% 128");
  MOE_CHECK_ARG(K > 0 && K % 128 == 0 && F > 0 && F % 128 == 0, "gemm_fwd_swiglu_mxq: K, F %% 128");
  MOE_CHECK_ARG(A && A_sc && B && B_sc && B3 && B3_sc && poff && aux,
                "gemm_fwd_swiglu_mxq: null pointer");
  MOE_CHECK_ARG(h_q && h_s && hT_q && hT_s && aligned16(h_q) && aligned16(hT_q),
                "gemm_fwd_swiglu_mxq: null or unaligned MX output");
  Params p = base_params(poff, E, dev_status);
  p.num_kb = K / 128;
  p.b_rows_per_e = K;
  p.a_sc = A_sc;
  p.a_sc_kchunks = K / 128;
  p.b_sc = B_sc;
  p.b3_sc = B3_sc;
  p.b_sc_kchunks = (int)((long long)E * K / 128);
  p.n_tiles = F / (BN / 2);
  p.ldc = F;
  p.aux = static_cast<__nv_bfloat16*>(aux);
  p.ld_aux = 2LL * F;
  p.half = F;
  p.quant = 1;
  p.q_sr = h_s;
  p.q_sc = hT_s;
  p.q_row_kchunks = F / 128;
  p.q_col_kchunks = A_pad_max / 128;
  Maps m;
  MOE_TRY(make_map(&m.a, A, 1, K, A_pad_max, 128, BM));
  p.b3d = make_map_mn3(&m.b, B, 1, F, (uint64_t)E * K, 128, (BN / 2) / 128) &&
          make_map_mn3(&m.b3, B3, 1, F, (uint64_t)E * K, 128, (BN / 2) / 128);
  if (!p.b3d) {
    MOE_TRY(make_map(&m.b, B, 1, F, (uint64_t)E * K, 128, 128));
    MOE_TRY(make_map(&m.b3, B3, 1, F, (uint64_t)E * K, 128, 128));
  }
  MOE_TRY(make_out_map(&m.c2, aux, 2ULL * F, A_pad_max));
  MOE_TRY(make_map(&m.qr, h_q, 1, F, A_pad_max, 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE));
  MOE_TRY(make_map(&m.qc, hT_q, 1, F, A_pad_max, 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE));
  m.q = true;
  m.c = m.in = m.a;
  const int max_tiles = (A_pad_max / BM) * p.n_tiles;
  return launch<true, false, B_MN_DUAL_N, EPI_SWIGLU>(m, p, max_tiles, s);
}

// MXFP8 GEMM2 dgrad with the SwiGLU-backward epilogue whose dA = [dA1 | dA3]
// [A_pad_max, 2K] leaves as MX codes: along the 2K columns (dA_q / dA_s,
// for the GEMM1 dgrad) and down the rows (dAT_q / dAT_s, for the GEMM1
// weight gradient), from the bf16-rounded dA.  dA itself is not stored.
extern "C" moe_status_t moe_grouped_gemm_dgrad_swiglu_mxq(
    const void* dC, const uint8_t* dC_sc, const void* B, const uint8_t* B_sc,
    const int32_t* poff, int E, int A_pad_max, int N, int K, const void* aux, uint8_t* dA_q,
    uint8_t* dA_s, uint8_t* dAT_q, uint8_t* dAT_s, int32_t* dev_status, moe_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  MOE_CHECK_ARG(E > 0 && E <= MAX_E, "gemm_dgrad_swiglu_mxq: E must be in [1, %d]", MAX_E);
  MOE_CHECK_ARG(A_pad_max > 0 && A_pad_max % 128 == 0, "gemm_dgrad_swiglu_mxq: A_pad_max %% 128");
  MOE_CHECK_ARG(N > 0 && N % 128 == 0 && K > 0 && K % 256 == 0,
                "gemm_dgrad_swiglu_mxq: N %% 128, K %% 256");
  MOE_CHECK_ARG(dC && dC_sc && B && B_sc && poff && aux, "gemm_dgrad_swiglu_mxq: null pointer");
  MOE_CHECK_ARG(dA_q && dA_s && dAT_q && dAT_s && aligned16(dA_q) && aligned16(dAT_q),
                "gemm_dgrad_swiglu_mxq: null or unaligned MX output");
  Params p = base_params(poff, E, dev_status);
  p.num_kb = N / 128;
  p.b_rows_per_e = K;
  p.k_split = N;
  p.n_tiles = K / BN;
  p.a_sc = dC_sc;
  p.a_sc_kchunks = N / 128;
  p.b_sc = B_sc;
  p.b_sc_kchunks = N / 128;
  p.aux = const_cast<__nv_bfloat16*>(static_cast<const __nv_bfloat16*>(aux));
  p.ld_aux = 2LL * K;
  p.half = K;
  p.ldc = 2LL * K;
  p.quant = 1;
  p.q_sr = dA_s;
  p.q_sc = dAT_s;
  p.q_row_kchunks = 2 * K / 128;
  p.q_col_kchunks = A_pad_max / 128;
  Maps m;
  MOE_TRY(make_map(&m.a, dC, 1, N, A_pad_max, 128, BM));
  MOE_TRY(make_map(&m.b, B, 1, N, (uint64_t)E * K, 128, BN));
  MOE_TRY(make_out_map(&m.in, aux, 2ULL * K, A_pad_max));
  MOE_TRY(make_map(&m.qr, dA_q, 1, 2ULL * K, A_pad_max, 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE));
  MOE_TRY(make_map(&m.qc, dAT_q, 1, 2ULL * K, A_pad_max, 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE));
  m.q = true;
  m.c = m.b3 = m.c2 = m.a;
  const int max_tiles = (A_pad_max / BM) * p.n_tiles;
  return launch<true, false, B_K, EPI_SWIGLU_BWD>(m, p, max_tiles, s);
}

extern "C" moe_status_t moe_grouped_gemm_dgrad(int dt, const void* dC, const uint8_t* dC_sc,
                                               const void* B, const uint8_t* B_sc,
                                               const void* B3, const uint8_t* B3_sc,
                                               const int32_t* poff, int E, int A_pad_max, int N,
                                               int K, int epilogue, const void* aux, void* dA,
                                               int32_t* dev_status, moe_stream_t stream) {
  return moe::grouped_gemm_dgrad(dt, dC, dC_sc, B, B_sc, B3, B3_sc, poff, E, A_pad_max, N, K,
                                 epilogue, aux, dA, nullptr, nullptr, dev_status,
                                 reinterpret_cast<cudaStream_t>(stream));
}

// moe_grouped_gemm_dgrad plus an optional rank-1 term in the EPI_NONE
// epilogue: dA[row, n] += row_scale[row] * col_vec[e * K + n] for the rows
// of group e (row_scale per padded row, col_vec [E, K] fp32, 16-byte
// aligned).  The layer backward adds the router's share of dx this way.
moe_status_t moe::grouped_gemm_dgrad(int dt, const void* dC, const uint8_t* dC_sc, const void* B,
                                     const uint8_t* B_sc, const void* B3, const uint8_t* B3_sc,
                                     const int32_t* poff, int E, int A_pad_max, int N, int K,
                                     int epilogue, const void* aux, void* dA,
                                     const float* row_scale, const float* col_vec,
                                     int32_t* dev_status, cudaStream_t s) {
  const bool mx = dt == MOE_MXFP8;
  MOE_CHECK_ARG(dt == MOE_BF16 || dt == MOE_MXFP8, "gemm_dgrad: bad dtype");
  MOE_CHECK_ARG(E > 0 && E <= MAX_E, "gemm_dgrad: E must be in [1, %d]", MAX_E);
  MOE_CHECK_ARG(A_pad_max > 0 && A_pad_max % 128 == 0, "gemm_dgrad: A_pad_max %% 128");
  MOE_CHECK_ARG(N > 0 && N % (mx ? 128 : 64) == 0, "gemm_dgrad: N %% %d", mx ? 128 : 64);
  MOE_CHECK_ARG(K > 0 && K % 256 == 0, "gemm_dgrad: K %% 256");
  MOE_CHECK_ARG(dC && B && dA && poff, "gemm_dgrad: null pointer");
  MOE_CHECK_ARG(!mx || (dC_sc && B_sc), "gemm_dgrad: MX needs scales");
  const int eb = mx ? 1 : 2;
  const bool dual = B3 != nullptr;
  MOE_CHECK_ARG(!dual || epilogue == MOE_EPI_NONE, "gemm_dgrad: B3 only with EPI_NONE");
  MOE_CHECK_ARG(!(dual && mx) || B3_sc, "gemm_dgrad: MX needs B3 scales");
  const int Ktot = dual ? 2 * N : N;    // reduction length over dC's columns
  Params p = base_params(poff, E, dev_status);
  p.num_kb = Ktot / (128 / eb);
  p.b_rows_per_e = K;
  p.k_split = N;
  p.n_tiles = K / BN;
  p.a_sc = dC_sc;
  p.a_sc_kchunks = Ktot / 128;
  p.b_sc = B_sc;
  p.b3_sc = B3_sc;
  p.b_sc_kchunks = N / 128;
  p.C = static_cast<__nv_bfloat16*>(dA);
  Maps m;
  MOE_TRY(make_map(&m.a, dC, eb, Ktot, A_pad_max, 128 / eb, BM));
  MOE_TRY(make_map(&m.b, B, eb, N, (uint64_t)E * K, 128 / eb, BN));
  const int max_tiles = (A_pad_max / BM) * p.n_tiles;
  if (epilogue == MOE_EPI_SWIGLU_BWD) {
    MOE_CHECK_ARG(aux != nullptr, "gemm_dgrad: SWIGLU_BWD needs aux = [H1|H3]");
    p.aux = const_cast<__nv_bfloat16*>(static_cast<const __nv_bfloat16*>(aux));
    p.ld_aux = 2LL * K;
    p.half = K;
    p.ldc = 2LL * K;
    MOE_TRY(make_out_map(&m.c, dA, 2ULL * K, A_pad_max));
    MOE_TRY(make_out_map(&m.in, aux, 2ULL * K, A_pad_max));
    m.b3 = m.c2 = m.a;
    return mx ? launch<true, false, B_K, EPI_SWIGLU_BWD>(m, p, max_tiles, s)
              : launch<false, false, B_K, EPI_SWIGLU_BWD>(m, p, max_tiles, s);
  }
  MOE_CHECK_ARG(epilogue == MOE_EPI_NONE, "gemm_dgrad: epilogue must be NONE or SWIGLU_BWD");
  MOE_CHECK_ARG((row_scale == nullptr) == (col_vec == nullptr) && (!col_vec || aligned16(col_vec)),
                "gemm_dgrad: row_scale and col_vec go together (col_vec 16-byte aligned)");
  p.row_scale = row_scale;
  p.col_vec = col_vec;
  p.col_ld = K;
  p.ldc = K;
  MOE_TRY(make_out_map(&m.c, dA, K, A_pad_max));
  m.c2 = m.in = m.a;
  if (!dual) {
    m.b3 = m.a;
    return mx ? launch<true, false, B_K, EPI_STORE>(m, p, max_tiles, s)
              : launch<false, false, B_K, EPI_STORE>(m, p, max_tiles, s);
  }
  MOE_TRY(make_map(&m.b3, B3, eb, N, (uint64_t)E * K, 128 / eb, BN));
  return mx ? launch<true, false, B_K_DUAL_K, EPI_STORE>(m, p, max_tiles, s)
            : launch<false, false, B_K_DUAL_K, EPI_STORE>(m, p, max_tiles, s);
}

extern "C" moe_status_t moe_grouped_gemm_wgrad(int dt, const void* A, const uint8_t* A_sc,
                                               const void* dC, const uint8_t* dC_sc,
                                               const int32_t* poff, int E, int A_pad_max, int K,
                                               int N, void* dB, void* dB3, int32_t* dev_status,
                                               moe_stream_t stream) {
  return moe::grouped_gemm_wgrad(dt, A, A_sc, dC, dC_sc, poff, nullptr, E, A_pad_max, K, N, dB,
                                 dB3, dev_status, reinterpret_cast<cudaStream_t>(stream));
}

// Weight-gradient grouped GEMM.  a_src == null: A is the permuted buffer
// [A_pad_max, K]; otherwise (BF16) A row r is x[a_src[r]] of the unpermuted
// x [a_rows, K] (zero where a_src[r] < 0), gathered by the producer.  The
// reduction of group e stops after its last real row when `offsets` (the
// unpadded group offsets) is given.
static moe_status_t wgrad_impl(int dt, const void* A, const uint8_t* A_sc, const void* dC,
                               const uint8_t* dC_sc, const int32_t* poff, const int32_t* offsets,
                               int E, int A_pad_max, int K, int N, void* dB, void* dB3,
                               const int32_t* a_src, int a_rows, int32_t* dev_status,
                               cudaStream_t s) {
  const bool mx = dt == MOE_MXFP8;
  const bool gather = a_src != nullptr;
  MOE_CHECK_ARG(dt == MOE_BF16 || dt == MOE_MXFP8, "gemm_wgrad: bad dtype");
  MOE_CHECK_ARG(!(gather && mx), "gemm_wgrad: row gathers are BF16 only");
  MOE_CHECK_ARG(!gather || (a_rows > 0 && aligned16(a_src) && aligned16(A)),
                "gemm_wgrad: gathered A needs T > 0 and 16-byte aligned x and src");
  MOE_CHECK_ARG(E > 0 && E <= MAX_E, "gemm_wgrad: E must be in [1, %d]", MAX_E);
  MOE_CHECK_ARG(A_pad_max > 0 && A_pad_max % 128 == 0, "gemm_wgrad: A_pad_max %% 128");
  MOE_CHECK_ARG(K > 0 && K % 128 == 0, "gemm_wgrad: K %% 128");
  MOE_CHECK_ARG(N > 0 && N % 256 == 0, "gemm_wgrad: N %% 256");
  MOE_CHECK_ARG(A && dC && dB && poff, "gemm_wgrad: null pointer");
  MOE_CHECK_ARG(!mx || (A_sc && dC_sc), "gemm_wgrad: MX needs scales");
#ifndef MOE_NO_PAIR_WGRAD
  // BF16 with 256-aligned weight shapes: 256 x 256 tiles on SM pairs (the
  // gathered form runs on single SMs: its cp.async copies signal a barrier
  // of their own CTA only)
  if (!mx && !gather && K % 256 == 0)
    return grouped_gemm_wgrad_pair(A, dC, poff, offsets, E, A_pad_max, K, N, dB, dB3, dev_status,
                                   s);
#endif
  const int eb = mx ? 1 : 2;
  const int Ncols = dB3 ? 2 * N : N;
  Params p = base_params(poff, E, dev_status);
  p.wgrad = 1;
  p.offsets = offsets;
  p.m_tiles_w = K / BM;
  p.n_tiles = Ncols / BN;
  p.k_out = K;
  p.a_sc = A_sc;
  p.a_sc_kchunks = A_pad_max / 128;
  p.b_sc = dC_sc;
  p.b_sc_kchunks = A_pad_max / 128;
  p.C = static_cast<__nv_bfloat16*>(dB);
  p.C2 = static_cast<__nv_bfloat16*>(dB3);
  p.n_split = dB3 ? N : 0;
  p.ldc = N;
  p.c_expert_stride = (long long)K * N;
  p.a_src = a_src;
  p.a_oob = a_rows;
  p.a_x = static_cast<const __nv_bfloat16*>(A);
  p.a_ld = K;
  Maps m;
  if (gather) {
    MOE_TRY(make_map(&m.a, A, 2, K, a_rows, 64, 1));   // unused by the gathering producer
  } else {
    p.a3d = make_map_mn3(&m.a, A, eb, K, A_pad_max, 128 / eb, BM * eb / 128);
    if (!p.a3d) MOE_TRY(make_map(&m.a, A, eb, K, A_pad_max, 128 / eb, 128 / eb));
  }
  p.b3d = make_map_mn3(&m.b, dC, eb, Ncols, A_pad_max, 128 / eb, BN * eb / 128);
  if (!p.b3d) {
    MOE_CHECK_ARG(!gather, "gemm_wgrad: gathered A needs the 3-D map of dC");
    MOE_TRY(make_map(&m.b, dC, eb, Ncols, A_pad_max, 128 / eb, 128 / eb));
  }
  MOE_TRY(make_out_map(&m.c, dB, N, (uint64_t)E * K));
  if (dB3) MOE_TRY(make_out_map(&m.c2, dB3, N, (uint64_t)E * K));
  else m.c2 = m.c;
  m.b3 = m.in = m.a;
  const int max_tiles = E * p.m_tiles_w * p.n_tiles;
  if (gather) return launch<false, true, B_MN, EPI_STORE, true>(m, p, max_tiles, s);
  return mx ? launch<true, true, B_MN, EPI_STORE>(m, p, max_tiles, s)
            : launch<false, true, B_MN, EPI_STORE>(m, p, max_tiles, s);
}

// moe_grouped_gemm_wgrad that stops each group's reduction after its last
// real row (offsets = the unpadded group offsets, E + 1 ints, or null):
// whole K blocks of zero padding rows are not loaded or multiplied.
moe_status_t moe::grouped_gemm_wgrad(int dt, const void* A, const uint8_t* A_sc, const void* dC,
                                     const uint8_t* dC_sc, const int32_t* poff,
                                     const int32_t* offsets, int E, int A_pad_max, int K, int N,
                                     void* dB, void* dB3, int32_t* dev_status, cudaStream_t s) {
  return wgrad_impl(dt, A, A_sc, dC, dC_sc, poff, offsets, E, A_pad_max, K, N, dB, dB3, nullptr,
                    0, dev_status, s);
}

extern "C" moe_status_t moe_grouped_gemm_wgrad_gather(const void* x, int T, const int32_t* src,
                                                      const void* dC, const int32_t* poff,
                                                      const int32_t* offsets, int E,
                                                      int A_pad_max, int K, int N, void* dB,
                                                      void* dB3, int32_t* dev_status,
                                                      moe_stream_t stream) {
  MOE_CHECK_ARG(x && src, "gemm_wgrad_gather: null x or src");
  return wgrad_impl(MOE_BF16, x, nullptr, dC, nullptr, poff, offsets, E, A_pad_max, K, N, dB,
                    dB3, src, T, dev_status, reinterpret_cast<cudaStream_t>(stream));
}
