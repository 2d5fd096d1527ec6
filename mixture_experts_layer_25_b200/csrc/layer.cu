// The whole MoE feed-forward layer, forward and backward, composed from the
// library's calls on one stream with no host synchronisation.
//
// Forward:  route -> GEMM1 + SwiGLU with the rowwise dispatch fused into
//           its producer (token rows gathered from x by src) -> GEMM2 ->
//           gate-weighted combine.  (MXFP8 and the tokens-N GEMMs take a
//           separate permute pass that writes Xp.)
// Backward: combine bwd (dY = g dout, dg, dl) -> GEMM2 dgrad fused with the
//           SwiGLU backward -> GEMM2 wgrad -> GEMM1 dgrad (+ the router's
//           share of dx as a rank-1 epilogue term) -> unpermute-sum (dx) ->
//           GEMM1 wgrad -> router weight grad (a host-buffer step downloads
//           dx under the last two).
// In MXFP8 mode every GEMM operand is quantised along that GEMM's K first
// (weights included, inside the step); operands used by two GEMMs with
// different K axes are quantised along both in one pass.  BF16 layers whose
// experts average fewer than 256 rows take the tokens-N kernel for the
// forward GEMMs and the GEMM1 dgrad (see tokens_n below).
#include <mutex>

#include "common.cuh"

namespace {

struct Layout {
  size_t off = 0;
  char* base = nullptr;
  template <class T>
  T* take(size_t count) {
    off = moe::round_up(off, 256);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
};

bool desc_ok(const moe_layer_desc* L) {
  if (!L) return false;
  if (L->T <= 0 || L->d <= 0 || L->E <= 0 || L->k <= 0 || L->F <= 0) return false;
  if (L->align != 128 || L->k > L->E || L->k > 16) return false;
  if (L->d % 256 || L->F % 256) return false;
  if (L->route_mode != MOE_ROUTE_ROUTER && L->route_mode != MOE_ROUTE_GIVEN) return false;
  if (L->dtype != MOE_BF16 && L->dtype != MOE_MXFP8) return false;
  if (L->route_mode == MOE_ROUTE_ROUTER && L->E > 512) return false;
  if (L->E > 1024) return false;
  return true;
}

int a_pad_max(const moe_layer_desc* L) {
  const long long a = (long long)L->T * L->k + (long long)L->E * (L->align - 1);
  return (int)((a + 127) / 128 * 128);
}

bool tokens_n(const moe_layer_desc* L);

// The BF16 layer on the main grouped GEMM reads the token rows straight
// from x (row gathers in the GEMM1 producers): no permuted copy Xp.
#ifndef MOE_GATHER_DISPATCH
#define MOE_GATHER_DISPATCH 0     // measured slower than the permute pass: off
#endif
bool gathers(const moe_layer_desc* L) {
  return MOE_GATHER_DISPATCH && L->dtype == MOE_BF16 && !tokens_n(L);
}

size_t layout(const moe_layer_desc* L, void* base, moe_ctx_view* v) {
  Layout l;
  l.base = static_cast<char*>(base);
  moe_ctx_view x{};
  const size_t T = L->T, d = L->d, E = L->E, k = L->k, F = L->F;
  const size_t A = a_pad_max(L);
  x.A_pad_max = (int)A;
  x.topk_idx = l.take<int32_t>(T * k);
  x.gates = l.take<float>(T * k);
  x.logits = L->route_mode == MOE_ROUTE_ROUTER ? l.take<float>(T * E) : nullptr;
  x.counts = l.take<int32_t>(E);
  x.offsets = l.take<int32_t>(E + 1);
  x.poff = l.take<int32_t>(E + 1);
  x.dst = l.take<int32_t>(T * k);
  x.src = l.take<int32_t>(A);
  x.dg = l.take<float>(T * k);
  x.dl = l.take<float>(T * k);
  x.dl_rows = l.take<float>(A);
  // the bf16 permuted copy: only BF16 layers that do not gather need it
  x.Xp = (L->dtype == MOE_BF16 && !gathers(L)) ? l.take<__nv_bfloat16>(A * d) : nullptr;
  x.H13 = l.take<__nv_bfloat16>(A * 2 * F);
  // MXFP8: h and dA13 leave their GEMM epilogues as MX codes only
  x.h = L->dtype == MOE_MXFP8 ? nullptr : l.take<__nv_bfloat16>(A * F);
  x.Y = l.take<__nv_bfloat16>(A * d);
  x.dXp = x.Y;   // Y is dead once the combine backward has run
  x.dY = L->dtype == MOE_MXFP8 ? nullptr : l.take<__nv_bfloat16>(A * d);
  x.dA13 = L->dtype == MOE_MXFP8 ? nullptr : l.take<__nv_bfloat16>(A * 2 * F);
  if (L->dtype == MOE_MXFP8) {
    x.Xp_q = l.take<uint8_t>(A * d);       x.Xp_s = l.take<uint8_t>(A * d / 32);
    x.W13_q = l.take<uint8_t>(2 * E * d * F); x.W13_s = l.take<uint8_t>(2 * E * d * F / 32);
    x.W2_q = l.take<uint8_t>(E * F * d);   x.W2_s = l.take<uint8_t>(E * F * d / 32);
    x.h_q = l.take<uint8_t>(A * F);        x.h_s = l.take<uint8_t>(A * F / 32);
    x.dY_q = l.take<uint8_t>(A * d);       x.dY_s = l.take<uint8_t>(A * d / 32);
    x.W2t_q = l.take<uint8_t>(E * F * d);  x.W2t_s = l.take<uint8_t>(E * F * d / 32);
    x.dA_q = l.take<uint8_t>(A * 2 * F);   x.dA_s = l.take<uint8_t>(A * 2 * F / 32);
    x.W13t_q = l.take<uint8_t>(2 * E * d * F); x.W13t_s = l.take<uint8_t>(2 * E * d * F / 32);
    x.hT_q = l.take<uint8_t>(A * F);       x.hT_s = l.take<uint8_t>(A * F / 32);
    x.dYT_q = l.take<uint8_t>(A * d);      x.dYT_s = l.take<uint8_t>(A * d / 32);
    x.XpT_q = l.take<uint8_t>(A * d);      x.XpT_s = l.take<uint8_t>(A * d / 32);
    x.dAT_q = l.take<uint8_t>(A * 2 * F);  x.dAT_s = l.take<uint8_t>(A * 2 * F / 32);
  }
  const size_t ws_route =
      moe_route_workspace_size(L->T, L->route_mode == MOE_ROUTE_ROUTER ? L->d : 0, L->E);
  const size_t ws_unperm = moe_unpermute_sum_workspace_size(L->d, L->E);
  const size_t ws_rw = moe_router_wgrad_workspace_size(L->d, (int)A);
  x.ws_bytes = ws_route > ws_unperm ? ws_route : ws_unperm;
  if (ws_rw > x.ws_bytes) x.ws_bytes = ws_rw;
  x.ws = l.take<uint8_t>(x.ws_bytes);
  if (v) *v = x;
  return moe::round_up(l.off, 256);
}

thread_local void* const* g_events = nullptr;
thread_local int g_nevents = 0;

// record the start (end = false) or end of stage s, if a benchmark asked
void mark(int s, bool end, cudaStream_t st) {
  const int i = 2 * s + (end ? 1 : 0);
  if (g_events && i < g_nevents && g_events[i])
    cudaEventRecord(static_cast<cudaEvent_t>(g_events[i]), st);
}

enum Stage { S_ROUTE, S_PERMUTE, S_QW, S_GEMM1, S_QH, S_GEMM2, S_COMBINE, S_COMBINE_BWD,
             S_QD2, S_DGRAD2, S_QW2, S_WGRAD2, S_QD1, S_DGRAD1, S_QW1, S_WGRAD1, S_UNPERMUTE,
             S_ROUTER_WGRAD };

}  // namespace

extern "C" void moe_set_stage_events(void* const* events, int n) {
  g_events = events;
  g_nevents = events ? n : 0;
}

using moe::set_error;

extern "C" size_t moe_layer_ctx_bytes(const moe_layer_desc* desc) {
  if (!desc_ok(desc)) return 0;
  return layout(desc, nullptr, nullptr);
}

extern "C" moe_status_t moe_layer_ctx_view(const moe_layer_desc* desc, void* ctx,
                                           moe_ctx_view* view) {
  MOE_CHECK_ARG(desc_ok(desc), "moe_layer_ctx_view: bad layer description");
  MOE_CHECK_ARG(ctx && view, "moe_layer_ctx_view: null pointer");
  layout(desc, ctx, view);
  return MOE_OK;
}

// The BF16 forward GEMMs and the GEMM1 dgrad take the tokens-N kernel when
// an expert gets fewer than 256 rows on average (T k < 256 E): the 128-row
// group padding is then a large share of the rows (about 64 of 171 at
// T = 8192, k = 8, E = 384), and multiplying only the real rows pays for
// that kernel's lower per-tile rate (measured: 12% faster layer at that
// shape, 6-7% slower at 512 rows per expert).
#ifndef MOE_TN_MIN_ROWS
#define MOE_TN_MIN_ROWS 256     // mean rows per expert below which the tokens-N kernel runs
#endif
namespace {
bool tokens_n(const moe_layer_desc* L) {
  return L->dtype == MOE_BF16 && (long long)L->T * L->k < (long long)MOE_TN_MIN_ROWS * L->E &&
         L->d % 128 == 0 && L->F % 64 == 0;
}
}  // namespace

static moe_status_t check_common(const moe_layer_desc* L, const moe_layer_weights* w, void* ctx,
                                 size_t ctx_bytes) {
  MOE_CHECK_ARG(desc_ok(L),
                "moe_layer: bad description (align 128, d %% 256, F %% 256, k <= min(E,16), "
                "router mode E <= 512, E <= 1024)");
  MOE_CHECK_ARG(w && w->W1 && w->W3 && w->W2, "moe_layer: missing expert weights");
  if (L->route_mode == MOE_ROUTE_ROUTER) MOE_CHECK_ARG(w->Wr, "moe_layer: router mode needs Wr");
  else MOE_CHECK_ARG(w->topk_idx && w->gates, "moe_layer: given mode needs topk_idx and gates");
  MOE_CHECK_ARG(ctx && (reinterpret_cast<uintptr_t>(ctx) & 255) == 0,
                "moe_layer: ctx must be 256-byte aligned");
  const size_t need = moe_layer_ctx_bytes(L);
  if (ctx_bytes < need) {
    set_error("moe_layer: ctx %zu < %zu bytes", ctx_bytes, need);
    return MOE_ERR_WORKSPACE;
  }
  return MOE_OK;
}

extern "C" moe_status_t moe_layer_fwd(const moe_layer_desc* L, const moe_layer_weights* w,
                                      const void* x, void* out, void* ctx, size_t ctx_bytes,
                                      int32_t* dev_status, moe_stream_t stream) {
  MOE_TRY(check_common(L, w, ctx, ctx_bytes));
  MOE_CHECK_ARG(x && out, "moe_layer_fwd: null x/out");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  moe_ctx_view c;
  layout(L, ctx, &c);
  const int T = L->T, d = L->d, E = L->E, k = L->k, F = L->F, A = c.A_pad_max;
  const bool mx = L->dtype == MOE_MXFP8;

  if (L->route_mode == MOE_ROUTE_GIVEN) {
    if (cudaMemcpyAsync(c.topk_idx, w->topk_idx, sizeof(int32_t) * T * k, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(c.gates, w->gates, sizeof(float) * T * k, cudaMemcpyDeviceToDevice, s) != cudaSuccess) {
      set_error("moe_layer_fwd: copy of the given routing failed");
      return MOE_ERR_CUDA;
    }
  }
  mark(S_ROUTE, false, s);
  MOE_TRY(moe_route(x, w->Wr, w->bias, T, d, E, k, L->align, L->route_mode, c.topk_idx, c.gates,
                    c.counts, c.offsets, c.poff, c.dst, c.src, A, c.logits, c.ws, c.ws_bytes,
                    dev_status, stream));
  mark(S_ROUTE, true, s);
  if (!mx) {
    if (!gathers(L)) {
      mark(S_PERMUTE, false, s);
      MOE_TRY(moe_permute(x, c.dst, c.offsets, c.poff, T, k, d, E, A, c.Xp, nullptr, nullptr,
                          stream));
      mark(S_PERMUTE, true, s);
    }
    mark(S_GEMM1, false, s);
    if (tokens_n(L))
      MOE_TRY(moe::gemm_tn(MOE_EPI_SWIGLU, c.Xp, w->W1, w->W3, 0, c.poff, c.offsets, E, A, F, d,
                           c.h, c.H13, nullptr, nullptr, dev_status, s));
    else if (gathers(L))   // dispatch fused into the GEMM: token rows gathered from x by src
      MOE_TRY(moe_grouped_gemm_fwd_gather(x, T, c.src, w->W1, w->W3, c.poff, E, A, F, d,
                                          MOE_EPI_SWIGLU, c.h, c.H13, dev_status, stream));
    else
      MOE_TRY(moe_grouped_gemm_fwd(MOE_BF16, c.Xp, nullptr, w->W1, nullptr, w->W3, nullptr,
                                   c.poff, E, A, F, d, MOE_EPI_SWIGLU, c.h, c.H13, dev_status,
                                   stream));
    mark(S_GEMM1, true, s);
    mark(S_GEMM2, false, s);
    if (tokens_n(L))
      MOE_TRY(moe::gemm_tn(MOE_EPI_NONE, c.h, w->W2, nullptr, 0, c.poff, c.offsets, E, A, d, F,
                           c.Y, nullptr, nullptr, nullptr, dev_status, s));
    else
      MOE_TRY(moe_grouped_gemm_fwd(MOE_BF16, c.h, nullptr, w->W2, nullptr, nullptr, nullptr,
                                   c.poff, E, A, d, F, MOE_EPI_NONE, c.Y, nullptr, dev_status,
                                   stream));
    mark(S_GEMM2, true, s);
  } else {
    const size_t wq = (size_t)E * d * F;
    uint8_t* W1q = c.W13_q; uint8_t* W3q = c.W13_q + wq;
    uint8_t* W1s = c.W13_s; uint8_t* W3s = c.W13_s + wq / 32;
    // rowwise dispatch straight into MX codes: along d (GEMM1) and down
    // the rows (GEMM1 weight gradient); no bf16 permuted copy
    mark(S_PERMUTE, false, s);
    MOE_TRY(moe_permute_mx(x, c.src, c.poff, T, d, E, A, c.Xp_q, c.Xp_s, c.XpT_q, c.XpT_s,
                           stream));
    mark(S_PERMUTE, true, s);
    // every weight along both K axes it is used with, in one pass each:
    // W1/W3 [E*d, F] down d (fwd GEMM1) and along F (GEMM1 dgrad); W2
    // [E*F, d] down F (fwd GEMM2) and along d (GEMM2 dgrad)
    mark(S_QW, false, s);
    MOE_TRY(mx_quantize_dual(w->W1, E * d, F, nullptr, c.W13t_q, c.W13t_s, W1q, W1s, stream));
    MOE_TRY(mx_quantize_dual(w->W3, E * d, F, nullptr, c.W13t_q + wq, c.W13t_s + wq / 32, W3q,
                             W3s, stream));
    MOE_TRY(mx_quantize_dual(w->W2, E * F, d, nullptr, c.W2t_q, c.W2t_s, c.W2_q, c.W2_s, stream));
    mark(S_QW, true, s);
    // GEMM1 + SwiGLU; its epilogue quantises h along F (fwd GEMM2) and down
    // the rows (GEMM2 wgrad) in place of storing it
    mark(S_GEMM1, false, s);
    MOE_TRY(moe_grouped_gemm_fwd_swiglu_mxq(c.Xp_q, c.Xp_s, W1q, W1s, W3q, W3s, c.poff, E, A, F,
                                            d, c.H13, c.h_q, c.h_s, c.hT_q, c.hT_s, dev_status,
                                            stream));
    mark(S_GEMM1, true, s);
    mark(S_GEMM2, false, s);
    MOE_TRY(moe_grouped_gemm_fwd(MOE_MXFP8, c.h_q, c.h_s, c.W2_q, c.W2_s, nullptr, nullptr, c.poff,
                                 E, A, d, F, MOE_EPI_NONE, c.Y, nullptr, dev_status, stream));
    mark(S_GEMM2, true, s);
  }
  mark(S_COMBINE, false, s);
  MOE_TRY(moe_unpermute_combine(c.Y, c.gates, c.dst, T, k, d, out, stream));
  mark(S_COMBINE, true, s);
  return MOE_OK;
}

namespace {

// moe_layer_bwd; dx_ready (nullable) is recorded on the stream once dx is
// complete, which is before the GEMM1 weight gradient and the router's
// weight gradient (a host-buffer step downloads dx under them)
moe_status_t layer_bwd(const moe_layer_desc* L, const moe_layer_weights* w, const void* x,
                       void* ctx, size_t ctx_bytes, const void* dout, void* dx,
                       moe_layer_grads* G, int32_t* dev_status, moe_stream_t stream,
                       cudaEvent_t dx_ready) {
  MOE_TRY(check_common(L, w, ctx, ctx_bytes));
  MOE_CHECK_ARG(x && dout && dx && G && G->dW1 && G->dW3 && G->dW2, "moe_layer_bwd: null pointer");
  const bool router = L->route_mode == MOE_ROUTE_ROUTER;
  moe_ctx_view c;
  layout(L, ctx, &c);
  const int T = L->T, d = L->d, E = L->E, k = L->k, F = L->F, A = c.A_pad_max;
  const bool mx = L->dtype == MOE_MXFP8;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // dx = the plain sum of each token's k rows of dXp: the router's share,
  // sum_j dl[t, j] W_r[:, e_j], was added to the rows of dXp by the GEMM1
  // dgrad epilogue.  Taken right after that dgrad, before the weight
  // gradients, which do not need it.
  auto dx_sum = [&]() -> moe_status_t {
    mark(S_UNPERMUTE, false, s);
    MOE_TRY(moe_unpermute_sum(c.dXp, c.dst, nullptr, nullptr, nullptr, T, k, d, E, dx, nullptr,
                              0, stream));
    mark(S_UNPERMUTE, true, s);
    if (dx_ready && cudaEventRecord(dx_ready, s) != cudaSuccess) {
      set_error("moe_layer_bwd: recording dx failed");
      return MOE_ERR_CUDA;
    }
    return MOE_OK;
  };
  // W_r^T [E, d] (fp32) in the workspace: the GEMM1 dgrad epilogue adds
  // dl_rows[r] * W_r[:, e] to each row r of expert e
  float* wrT = router ? static_cast<float*>(c.ws) : nullptr;
  // dg, dl, dl_rows (and in BF16 the gate-scaled rows dY)
  mark(S_COMBINE_BWD, false, s);
  MOE_TRY(moe_combine_bwd(dout, c.Y, c.gates, c.dst, c.offsets, c.poff, T, k, d, E,
                          mx ? nullptr : c.dY, c.dg, router ? c.dl : nullptr,
                          router ? c.dl_rows : nullptr, stream));
  mark(S_COMBINE_BWD, true, s);
  if (!mx) {
    mark(S_DGRAD2, false, s);
    MOE_TRY(moe_grouped_gemm_dgrad(MOE_BF16, c.dY, nullptr, w->W2, nullptr, nullptr, nullptr,
                                   c.poff, E, A, d, F, MOE_EPI_SWIGLU_BWD, c.H13, c.dA13,
                                   dev_status, stream));
    mark(S_DGRAD2, true, s);
    mark(S_WGRAD2, false, s);
    MOE_TRY(moe::grouped_gemm_wgrad(MOE_BF16, c.h, nullptr, c.dY, nullptr, c.poff, c.offsets, E,
                                    A, F, d, G->dW2, nullptr, dev_status, s));
    mark(S_WGRAD2, true, s);
    mark(S_DGRAD1, false, s);
    if (router) MOE_TRY(moe::transpose_f32(w->Wr, d, E, wrT, s));
    if (tokens_n(L))
      MOE_TRY(moe::gemm_tn(MOE_EPI_NONE, c.dA13, w->W1, w->W3, 1, c.poff, c.offsets, E, A, d,
                           2 * F, c.dXp, nullptr, router ? c.dl_rows : nullptr,
                           router ? wrT : nullptr, dev_status, s));
    else
      MOE_TRY(moe::grouped_gemm_dgrad(MOE_BF16, c.dA13, nullptr, w->W1, nullptr, w->W3, nullptr,
                                      c.poff, E, A, F, d, MOE_EPI_NONE, nullptr, c.dXp,
                                      router ? c.dl_rows : nullptr, router ? wrT : nullptr,
                                      dev_status, s));
    mark(S_DGRAD1, true, s);
    MOE_TRY(dx_sum());
    mark(S_WGRAD1, false, s);
    if (gathers(L))
      MOE_TRY(moe_grouped_gemm_wgrad_gather(x, T, c.src, c.dA13, c.poff, c.offsets, E, A, d, F,
                                            G->dW1, G->dW3, dev_status, stream));
    else
      MOE_TRY(moe::grouped_gemm_wgrad(MOE_BF16, c.Xp, nullptr, c.dA13, nullptr, c.poff,
                                      c.offsets, E, A, d, F, G->dW1, G->dW3, dev_status, s));
    mark(S_WGRAD1, true, s);
  } else {
    const size_t wq = (size_t)E * d * F;
    // (weights were quantised along both axes in the forward)
    // the gate-scaled rows dY straight into MX codes, along d (GEMM2 dgrad)
    // and down the rows (GEMM2 wgrad)
    mark(S_QD2, false, s);
    MOE_TRY(moe_combine_bwd_mx(dout, c.gates, c.topk_idx, c.src, c.poff, T, k, d, E, A, c.dY_q,
                               c.dY_s, c.dYT_q, c.dYT_s, stream));
    mark(S_QD2, true, s);
    // GEMM2 dgrad + SwiGLU backward; its epilogue quantises dA13 along 2F
    // (GEMM1 dgrad) and down the rows (GEMM1 wgrad) in place of storing it
    mark(S_DGRAD2, false, s);
    MOE_TRY(moe_grouped_gemm_dgrad_swiglu_mxq(c.dY_q, c.dY_s, c.W2t_q, c.W2t_s, c.poff, E, A, d, F,
                                              c.H13, c.dA_q, c.dA_s, c.dAT_q, c.dAT_s, dev_status,
                                              stream));
    mark(S_DGRAD2, true, s);
    mark(S_WGRAD2, false, s);
    MOE_TRY(moe::grouped_gemm_wgrad(MOE_MXFP8, c.hT_q, c.hT_s, c.dYT_q, c.dYT_s, c.poff,
                                    c.offsets, E, A, F, d, G->dW2, nullptr, dev_status, s));
    mark(S_WGRAD2, true, s);
    mark(S_DGRAD1, false, s);
    if (router) MOE_TRY(moe::transpose_f32(w->Wr, d, E, wrT, s));
    MOE_TRY(moe::grouped_gemm_dgrad(MOE_MXFP8, c.dA_q, c.dA_s, c.W13t_q, c.W13t_s, c.W13t_q + wq,
                               c.W13t_s + wq / 32, c.poff, E, A, F, d, MOE_EPI_NONE, nullptr,
                               c.dXp, router ? c.dl_rows : nullptr, router ? wrT : nullptr,
                               dev_status, s));
    mark(S_DGRAD1, true, s);
    MOE_TRY(dx_sum());
    mark(S_WGRAD1, false, s);
    MOE_TRY(moe::grouped_gemm_wgrad(MOE_MXFP8, c.XpT_q, c.XpT_s, c.dAT_q, c.dAT_s, c.poff,
                                    c.offsets, E, A, d, F, G->dW1, G->dW3, dev_status, s));
    mark(S_WGRAD1, true, s);
  }
  if (router && G->dWr) {
    mark(S_ROUTER_WGRAD, false, s);
    MOE_TRY(moe_router_wgrad(x, c.src, c.dl_rows, c.offsets, c.poff, T, d, E, A, G->dWr, c.ws,
                             c.ws_bytes, stream));
    mark(S_ROUTER_WGRAD, true, s);
  }
  return MOE_OK;
}

}  // namespace

extern "C" moe_status_t moe_layer_bwd(const moe_layer_desc* L, const moe_layer_weights* w,
                                      const void* x, void* ctx, size_t ctx_bytes,
                                      const void* dout, void* dx, moe_layer_grads* G,
                                      int32_t* dev_status, moe_stream_t stream) {
  return layer_bwd(L, w, x, ctx, ctx_bytes, dout, dx, G, dev_status, stream, nullptr);
}

namespace {

constexpr int kMaxCopyDevices = 64;
std::mutex g_copy_mu;
cudaStream_t g_copy_stream[2][kMaxCopyDevices] = {};   // [0]: uploads, [1]: downloads

// The library's copy streams on the current device (non-blocking, created
// on first use and kept until the process exits): uploads and downloads on
// separate streams, so that one call's uploads never queue behind the
// previous call's downloads.
moe_status_t copy_streams(cudaStream_t* up, cudaStream_t* down, int* dev_out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxCopyDevices) {
    set_error("moe_layer_step_host: no usable current device");
    return MOE_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_copy_mu);
  for (int i = 0; i < 2; ++i)
    if (!g_copy_stream[i][dev] &&
        cudaStreamCreateWithFlags(&g_copy_stream[i][dev], cudaStreamNonBlocking) != cudaSuccess) {
      g_copy_stream[i][dev] = nullptr;
      set_error("moe_layer_step_host: copy stream creation failed");
      return MOE_ERR_CUDA;
    }
  *up = g_copy_stream[0][dev];
  *down = g_copy_stream[1][dev];
  *dev_out = dev;
  return MOE_OK;
}

// Device input buffers of earlier host-buffer steps, each with the event
// after which that step was done reading it.  An upload into a known buffer
// waits only for that event, so a call given the other of two alternating
// buffer sets uploads its inputs under the previous call's backward; an
// unknown buffer waits for all work already on the caller's stream.
struct BufDone {
  int dev = -1;
  const void* ptr = nullptr;
  cudaEvent_t ev = nullptr;
};
constexpr int kBufSlots = 32;
std::mutex g_buf_mu;
BufDone g_buf[kBufSlots];
int g_buf_next = 0;

// q waits until buffer p of device dev is free; false if p is unknown
bool wait_buf(cudaStream_t q, int dev, const void* p, bool* ok) {
  std::lock_guard<std::mutex> lock(g_buf_mu);
  for (BufDone& b : g_buf)
    if (b.ev && b.dev == dev && b.ptr == p) {
      *ok = cudaStreamWaitEvent(q, b.ev, 0) == cudaSuccess;
      return true;
    }
  return false;
}

// records on q the point after which buffer p is free (the slot owns the event)
bool mark_buf(cudaStream_t q, int dev, const void* p) {
  cudaEvent_t ev = nullptr;
  if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) return false;
  if (cudaEventRecord(ev, q) != cudaSuccess) {
    cudaEventDestroy(ev);
    return false;
  }
  std::lock_guard<std::mutex> lock(g_buf_mu);
  BufDone* slot = nullptr;
  for (BufDone& b : g_buf)
    if (b.ev && b.dev == dev && b.ptr == p) slot = &b;
  if (!slot) {
    slot = &g_buf[g_buf_next];
    g_buf_next = (g_buf_next + 1) % kBufSlots;
  }
  if (slot->ev) cudaEventDestroy(slot->ev);   // every wait on it is already enqueued
  *slot = BufDone{dev, p, ev};
  return true;
}

struct Events {
  cudaEvent_t ev[4] = {};
  ~Events() {
    for (cudaEvent_t e : ev)
      if (e) cudaEventDestroy(e);   // released by the driver once the event has completed
  }
};

}  // namespace

// Schedule (s = the caller's stream; up / down = the library's upload and
// download streams; buffer events from the registry above):
//   up:   wait x_dev, dout_dev free | H2D x, dout | record in
//   s:    wait out_dev, dx_dev free | wait in | fwd | record fwd_done | bwd
//         (records dx_ready after the dx sum) | x_dev, dout_dev free
//   down: wait fwd_done | D2H out | out_dev free | wait dx_ready | D2H dx |
//         dx_dev free
// s never waits for the downloads: the next step's forward runs under this
// step's downloads when it has the other set of device buffers.  The host
// outputs are complete once s has been made to wait for the downloads
// (moe_layer_step_host_sync) and then synchronised.
extern "C" moe_status_t moe_layer_step_host(const moe_layer_desc* L, const moe_layer_weights* w,
                                            const void* x_host, const void* dout_host,
                                            void* out_host, void* dx_host, void* x_dev,
                                            void* dout_dev, void* out_dev, void* dx_dev,
                                            void* ctx, size_t ctx_bytes, moe_layer_grads* G,
                                            int32_t* dev_status, moe_stream_t stream) {
  MOE_TRY(check_common(L, w, ctx, ctx_bytes));
  MOE_CHECK_ARG(x_host && dout_host && out_host && dx_host && x_dev && dout_dev && out_dev && dx_dev,
                "moe_layer_step_host: null pointer");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaStream_t up = nullptr, down = nullptr;
  int dev = -1;
  MOE_TRY(copy_streams(&up, &down, &dev));
  Events E;
  for (cudaEvent_t& e : E.ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      e = nullptr;
      set_error("moe_layer_step_host: event creation failed");
      return MOE_ERR_CUDA;
    }
  cudaEvent_t start = E.ev[0], in = E.ev[1], fwd_done = E.ev[2], dx_ready = E.ev[3];
  const size_t bytes = (size_t)L->T * L->d * 2;
  auto fail = [](const char* what) {
    set_error("moe_layer_step_host: %s failed", what);
    return MOE_ERR_CUDA;
  };
  // uploads: each input buffer once the step that last read it is done
  // with it (or, for a buffer not seen before, after the caller's stream)
  bool ok = cudaEventRecord(start, s) == cudaSuccess;
  for (const void* p : {static_cast<const void*>(x_dev), static_cast<const void*>(dout_dev)}) {
    bool waited = true;
    if (ok && !wait_buf(up, dev, p, &waited)) waited = cudaStreamWaitEvent(up, start, 0) == cudaSuccess;
    ok = ok && waited;
  }
  if (!ok) return fail("ordering the uploads");
  if (cudaMemcpyAsync(x_dev, x_host, bytes, cudaMemcpyHostToDevice, up) != cudaSuccess ||
      cudaMemcpyAsync(dout_dev, dout_host, bytes, cudaMemcpyHostToDevice, up) != cudaSuccess ||
      cudaEventRecord(in, up) != cudaSuccess || cudaStreamWaitEvent(s, in, 0) != cudaSuccess)
    return fail("host-to-device copy of x and dout");
  // outputs: a device output buffer is rewritten only after the download
  // that last read it
  for (const void* p : {static_cast<const void*>(out_dev), static_cast<const void*>(dx_dev)}) {
    bool waited = true;
    if (wait_buf(s, dev, p, &waited) && !waited) return fail("ordering the output buffers");
  }
  moe_status_t st = moe_layer_fwd(L, w, x_dev, out_dev, ctx, ctx_bytes, dev_status, stream);
  const bool rec = cudaEventRecord(fwd_done, s) == cudaSuccess;
  const bool waited = rec && cudaStreamWaitEvent(down, fwd_done, 0) == cudaSuccess;
  bool copied_out = false;
  if (st == MOE_OK && waited)
    copied_out = cudaMemcpyAsync(out_host, out_dev, bytes, cudaMemcpyDeviceToHost, down) == cudaSuccess &&
                 mark_buf(down, dev, out_dev);
  // the backward records dx_ready before its last weight gradients: dx moves
  // to the host under them
  if (st == MOE_OK)
    st = layer_bwd(L, w, x_dev, ctx, ctx_bytes, dout_dev, dx_dev, G, dev_status, stream, dx_ready);
  bool copied_dx = false;
  if (st == MOE_OK && cudaStreamWaitEvent(down, dx_ready, 0) == cudaSuccess)
    copied_dx = cudaMemcpyAsync(dx_host, dx_dev, bytes, cudaMemcpyDeviceToHost, down) == cudaSuccess &&
                mark_buf(down, dev, dx_dev);
  // x and dout are read until the end of the backward
  if (st == MOE_OK && !(mark_buf(s, dev, x_dev) && mark_buf(s, dev, dout_dev)))
    st = fail("recording the input buffers' release");
  if (st == MOE_OK && !(waited && copied_out)) st = fail("device-to-host copy of out");
  if (st == MOE_OK && !copied_dx) st = fail("device-to-host copy of dx");
  return st;
}

extern "C" moe_status_t moe_layer_step_host_sync(moe_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaStream_t up = nullptr, down = nullptr;
  int dev = -1;
  MOE_TRY(copy_streams(&up, &down, &dev));
  cudaEvent_t ev = nullptr;
  if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) {
    set_error("moe_layer_step_host_sync: event creation failed");
    return MOE_ERR_CUDA;
  }
  const bool ok = cudaEventRecord(ev, down) == cudaSuccess && cudaStreamWaitEvent(s, ev, 0) == cudaSuccess;
  cudaEventDestroy(ev);   // released by the driver once the event has completed
  if (!ok) {
    set_error("moe_layer_step_host_sync: ordering the stream after the downloads failed");
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
