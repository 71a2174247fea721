// The C ABI declared in include/moe.h: plan (shape validation, workspace
// layout), argument checks, and the launch sequence of one MoE-layer forward
// pass on one stream.  No allocation, no host synchronisation, no
// device-to-host copy on the forward path.
#include <string.h>

#include <new>

#include "moe_internal.cuh"

#define MOE_EXPORT extern "C" __attribute__((visibility("default")))

struct moe_plan_s {
  moe_config cfg;
  size_t ws_bytes;
  int imax;          // max(I, Is)
  int ks_max;        // top_k_max + S
  size_t r_cap;      // max_tokens * ks_max rows
  // byte offsets inside the workspace
  size_t off_status, off_goff, off_done, off_wsplit, off_rscratch, off_partial, off_logits,
      off_ids, off_w, off_perm,
      off_inv, off_rowtok, off_xp, off_sx, off_h, off_sh, off_y;
  unsigned long long wait_limit_ns;
  int device;
  int num_sms;
};

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

thread_local cudaError_t g_last_cuda_error = cudaSuccess;

moe_status check_launch(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  g_last_cuda_error = e;
  return MOE_ERR_CUDA;
}

moe_status ensure_device(moe_plan_s* p) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (p->device == dev) return MOE_OK;
  static unsigned long long prepared_mask = 0;   // devices whose kernel attributes are set
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) return MOE_ERR_UNSUPPORTED;   // built for sm_100a only
  if (dev < 64 && !((prepared_mask >> dev) & 1ull)) {
    if (check_launch(moe::prepare_grouped_gemm_kernels()) != MOE_OK ||
        check_launch(moe::prepare_grouped_gemm_fp8_kernels()) != MOE_OK ||
        check_launch(moe::prepare_router_kernel()) != MOE_OK)
      return MOE_ERR_CUDA;
    prepared_mask |= 1ull << dev;
  }
  p->num_sms = sms;
  p->device = dev;
  return MOE_OK;
}

void record(moe_debug* dbg, int i, cudaStream_t st) {
  if (dbg != nullptr && dbg->events[i] != nullptr)
    cudaEventRecord(static_cast<cudaEvent_t>(dbg->events[i]), st);
}

moe_status check_common(const moe_plan_s* p, int T, int k, const void* workspace,
                        size_t ws_bytes) {
  if (p == nullptr) return MOE_ERR_INVALID_ARG;
  if (T < 0 || T > p->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
  if (k < 1 || k > p->cfg.top_k_max) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
    return MOE_ERR_INVALID_ARG;
  if (ws_bytes < p->ws_bytes) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

}  // namespace

MOE_EXPORT const char* moe_last_cuda_error_string(void) {
  return cudaGetErrorString(g_last_cuda_error);
}

MOE_EXPORT const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape, type or device";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_DEVICE: return "device-side failure (see status bits)";
  }
  return "unknown status";
}

MOE_EXPORT moe_status moe_plan_create(const moe_config* cfg, moe_plan_t* plan,
                                      size_t* workspace_bytes) {
  if (cfg == nullptr || plan == nullptr || workspace_bytes == nullptr) return MOE_ERR_INVALID_ARG;
  *plan = nullptr;
  const moe_config c = *cfg;
  if (c.max_tokens < 1 || c.hidden < 1 || c.num_experts < 1 || c.top_k_max < 1 || c.inter < 1)
    return MOE_ERR_INVALID_ARG;
  if (c.num_shared != 0 && c.num_shared != 1) return MOE_ERR_INVALID_ARG;
  if (c.renormalize != 0 && c.renormalize != 1) return MOE_ERR_INVALID_ARG;
  if (c.wtype != MOE_W_BF16 && c.wtype != MOE_W_FP8_E4M3_B128) return MOE_ERR_INVALID_ARG;
  if (c.top_k_max > c.num_experts) return MOE_ERR_INVALID_ARG;
  if (c.num_shared == 1 && c.shared_inter < 1) return MOE_ERR_INVALID_ARG;
  if (c.num_experts > moe::kMaxExperts || c.top_k_max > moe::kMaxTopK) return MOE_ERR_UNSUPPORTED;
  if (c.hidden % 128 != 0 || c.inter % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (c.num_shared == 1 && c.shared_inter % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (c.hidden > 65536 || c.inter > 65536 || c.shared_inter > 65536) return MOE_ERR_UNSUPPORTED;
  const int S = c.num_shared;
  const int imax = S && c.shared_inter > c.inter ? c.shared_inter : c.inter;
  const size_t T = (size_t)c.max_tokens, E = (size_t)c.num_experts, H = (size_t)c.hidden;
  const size_t ks = (size_t)c.top_k_max + S;
  const size_t r_cap = T * ks;
  if (r_cap > (size_t)0x7fffffff / 2) return MOE_ERR_UNSUPPORTED;

  moe_plan_s* p = new (std::nothrow) moe_plan_s();
  if (p == nullptr) return MOE_ERR_INVALID_ARG;
  p->cfg = c;
  p->imax = imax;
  p->ks_max = (int)ks;
  p->r_cap = r_cap;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes);
    return o;
  };
  p->off_status = take(64);
  p->off_goff = take(sizeof(int) * (E + 2));
  p->off_done = take(sizeof(unsigned int) * (E + 2));
  p->off_wsplit = take(2 * 3 * (size_t)moe::router_padded_experts((int)E) * H);
  p->off_rscratch = take(sizeof(int) * (size_t)moe::route_scratch_ints((int)T, (int)E));
  p->off_partial = take(sizeof(float) * (size_t)moe::router_partial_rows((int)T) * E);
  p->off_logits = take(sizeof(float) * T * E);
  p->off_ids = take(sizeof(int) * T * c.top_k_max);
  p->off_w = take(sizeof(float) * T * c.top_k_max);
  p->off_perm = take(sizeof(int) * T * c.top_k_max);
  p->off_inv = take(sizeof(int) * T * ks);
  p->off_rowtok = take(sizeof(int) * r_cap);
  if (c.wtype == MOE_W_BF16) {
    // bf16 permuted rows; h as two bf16 parts a row (rows 2r, 2r + 1); fp32 expert outputs
    p->off_xp = take(2 * r_cap * H);
    p->off_sx = 0;
    p->off_h = take(2 * 2 * r_cap * (size_t)imax);
    p->off_sh = 0;
    p->off_y = take(sizeof(float) * r_cap * H);
  } else {
    // e4m3 permuted rows and h with transposed 1x128 scales; bf16 expert outputs
    p->off_xp = take(r_cap * H);
    p->off_sx = take(sizeof(float) * (H / 128) * r_cap);
    p->off_h = take(r_cap * (size_t)imax);
    p->off_sh = take(sizeof(float) * ((size_t)imax / 128) * r_cap);
    p->off_y = take(2 * r_cap * H);
  }
  p->ws_bytes = off;
  p->wait_limit_ns = 2000000000ull;
  p->device = -1;
  p->num_sms = 0;
  *plan = p;
  *workspace_bytes = p->ws_bytes;
  return MOE_OK;
}

MOE_EXPORT void moe_plan_destroy(moe_plan_t plan) { delete plan; }

MOE_EXPORT moe_status moe_plan_set_wait_limit(moe_plan_t plan, uint64_t limit_ns) {
  if (plan == nullptr) return MOE_ERR_INVALID_ARG;
  plan->wait_limit_ns = limit_ns;
  return MOE_OK;
}

MOE_EXPORT size_t moe_router_split_bytes(moe_plan_t plan) {
  if (plan == nullptr) return 0;
  return (size_t)2 * 3 * (size_t)moe::router_padded_experts(plan->cfg.num_experts) *
         (size_t)plan->cfg.hidden;
}

MOE_EXPORT moe_status moe_split_router_weights(moe_plan_t plan, const float* router_w,
                                               void* split, size_t split_bytes, void* stream) {
  if (plan == nullptr || router_w == nullptr || split == nullptr || !aligned16(router_w) ||
      !aligned16(split))
    return MOE_ERR_INVALID_ARG;
  if (split_bytes < moe_router_split_bytes(plan)) return MOE_ERR_WORKSPACE;
  moe_status s = ensure_device(plan);
  if (s != MOE_OK) return s;
  return check_launch(moe::launch_split_router_weights(
      router_w, plan->cfg.num_experts, plan->cfg.hidden, static_cast<__nv_bfloat16*>(split),
      plan->num_sms, static_cast<cudaStream_t>(stream)));
}

// The forward pass; `co` says where the combine writes (the bf16 output, or
// fp32 partial rows of a tensor- / expert-parallel rank), and [eb, ee) which
// routed experts this call computes (their weights are the ones given).
// Argument checks common to the entry points are here; each entry point checks
// its own output arguments first.
static moe_status forward_impl(moe_plan_t plan, const moe_weights* wts, const void* hidden,
                               const uint8_t* valid, int T, int k, const moe::CombineOut& co,
                               int eb, int ee, void* workspace, size_t ws_bytes, void* stream,
                               moe_debug* dbg, const moe::SendArgs* send = nullptr) {
  moe_status s = check_common(plan, T, k, workspace, ws_bytes);
  if (s != MOE_OK) return s;
  if (wts == nullptr) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  const moe_config& c = plan->cfg;
  const int S = c.num_shared;
  if (hidden == nullptr || wts->router_w == nullptr || wts->w_gate_up == nullptr ||
      wts->w_down == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (S && (wts->ws_gate_up == nullptr || wts->ws_down == nullptr)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(hidden) || !aligned16(wts->router_w) ||
      !aligned16(wts->w_gate_up) || !aligned16(wts->w_down) ||
      (S && (!aligned16(wts->ws_gate_up) || !aligned16(wts->ws_down))))
    return MOE_ERR_INVALID_ARG;
  if ((wts->router_b != nullptr && (reinterpret_cast<uintptr_t>(wts->router_b) & 3u)) != 0)
    return MOE_ERR_INVALID_ARG;
  if (wts->router_split != nullptr && !aligned16(wts->router_split)) return MOE_ERR_INVALID_ARG;
  if (c.wtype == MOE_W_FP8_E4M3_B128 &&
      (wts->s_gate_up == nullptr || wts->s_down == nullptr ||
       (S && (wts->ss_gate_up == nullptr || wts->ss_down == nullptr))))
    return MOE_ERR_INVALID_ARG;
  s = ensure_device(plan);
  if (s != MOE_OK) return s;
  if (send != nullptr && (send->n_send < 1 || send->n_send >= plan->num_sms))
    return MOE_ERR_INVALID_ARG;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int E = c.num_experts, H = c.hidden, I = c.inter, Is = S ? c.shared_inter : 0;
  const int G = E + S;
  const int ks = k + S;
  const int R_cap = T * ks;
  unsigned int* status = at<unsigned int>(workspace, plan->off_status);
  int* goff = at<int>(workspace, plan->off_goff);
  float* partial = at<float>(workspace, plan->off_partial);
  float* logits = at<float>(workspace, plan->off_logits);
  int* ids = at<int>(workspace, plan->off_ids);
  float* w = at<float>(workspace, plan->off_w);
  int* perm = at<int>(workspace, plan->off_perm);
  int* inv = at<int>(workspace, plan->off_inv);
  int* rowtok = at<int>(workspace, plan->off_rowtok);
  auto* xp = at<__nv_bfloat16>(workspace, plan->off_xp);
  auto* h = at<__nv_bfloat16>(workspace, plan->off_h);
  float* y = at<float>(workspace, plan->off_y);
  const auto* x = static_cast<const __nv_bfloat16*>(hidden);

  record(dbg, 0, st);
  if (cudaMemsetAsync(status, 0, sizeof(unsigned int), st) != cudaSuccess) return MOE_ERR_CUDA;
  int splits = 1, kb_per_split = H / 64;
  moe::router_split_plan(T, E, H, plan->num_sms, moe::router_partial_rows(c.max_tokens),
                         &splits, &kb_per_split);
  // the router weights' bf16 split: the caller's (written once by
  // moe_split_router_weights), else made here in the workspace
  const __nv_bfloat16* w3 = static_cast<const __nv_bfloat16*>(wts->router_split);
  if (w3 == nullptr) {
    auto* w3_ws = at<__nv_bfloat16>(workspace, plan->off_wsplit);
    s = check_launch(moe::launch_split_router_weights(wts->router_w, E, H, w3_ws, plan->num_sms, st));
    if (s != MOE_OK) return s;
    w3 = w3_ws;
  }
  s = check_launch(moe::launch_router_logits_tc(x, valid, T, H, w3, E, partial, splits,
                                                kb_per_split, status, st));
  if (s != MOE_OK) return s;
  record(dbg, 1, st);
  s = check_launch(moe::launch_topk(partial, splits, wts->router_b, valid, T, E, k, c.renormalize,
                                    dbg != nullptr && dbg->logits != nullptr ? logits : nullptr,
                                    ids, w, st));
  if (s != MOE_OK) return s;
  record(dbg, 2, st);
  s = check_launch(moe::launch_route(ids, valid, T, E, k, S, eb, ee, goff, perm, inv, rowtok,
                                     status, at<int>(workspace, plan->off_rscratch), st));
  if (s != MOE_OK) return s;
  record(dbg, 3, st);
  const bool fp8 = c.wtype == MOE_W_FP8_E4M3_B128;
  if (!fp8) {
    s = check_launch(
        moe::launch_gather_rows(x, H, rowtok, goff + G, R_cap, xp, plan->num_sms, st));
  } else {
    s = check_launch(moe::launch_quant_scatter(x, valid, T, H, inv, ks,
                                               at<uint8_t>(workspace, plan->off_xp),
                                               at<float>(workspace, plan->off_sx),
                                               plan->num_sms, st));
  }
  if (s != MOE_OK) return s;
  record(dbg, 4, st);

  if (!fp8) {
    moe::GroupedGemmArgs ga;
    memset(&ga, 0, sizeof(ga));
    ga.a_routed = wts->w_gate_up;
    ga.a_shared = S ? wts->ws_gate_up : nullptr;
    ga.b = xp;
    ga.d = h;
    ga.group_offsets = goff;
    ga.E = E;
    ga.e_base = eb;
    ga.n_local = ee - eb;
    ga.G = G;
    ga.K_routed = H;
    ga.K_shared = H;
    ga.K_ld = H;
    ga.rows_per_expert = 2 * I;
    ga.m_tiles_routed = I / 128;
    ga.m_tiles_shared = S ? Is / 128 : 0;
    ga.up_routed = I;
    ga.up_shared = Is;
    ga.ldd = plan->imax;
    ga.R_cap = R_cap;
    ga.gated = true;
    ga.status = status;
    ga.timeout_bit = MOE_DEV_WAIT_TIMEOUT_GATE_UP;
    ga.wait_limit_ns = plan->wait_limit_ns;
    ga.num_ctas = plan->num_sms;
    s = check_launch(moe::launch_grouped_gemm(ga, st));
    if (s != MOE_OK) return s;
    record(dbg, 5, st);

    ga.a_routed = wts->w_down;
    ga.a_shared = S ? wts->ws_down : nullptr;
    ga.b = h;
    ga.d = y;
    ga.K_routed = I;
    ga.K_shared = S ? Is : 0;
    ga.K_ld = plan->imax;
    ga.rows_per_expert = H;
    ga.m_tiles_routed = H / 128;
    ga.m_tiles_shared = S ? H / 128 : 0;
    ga.up_routed = 0;
    ga.up_shared = 0;
    ga.ldd = H;
    ga.gated = false;
    ga.timeout_bit = MOE_DEV_WAIT_TIMEOUT_DOWN;
    if (send != nullptr) {
      ga.send = *send;
      ga.send.perm = perm;
      ga.send.row_token = rowtok;
      ga.send.done = at<unsigned int>(workspace, plan->off_done);
      if (cudaMemsetAsync(ga.send.done, 0, sizeof(unsigned int) * G, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
    s = check_launch(moe::launch_grouped_gemm(ga, st));
    if (s != MOE_OK) return s;
    record(dbg, 6, st);

    if (send == nullptr) s = check_launch(moe::launch_combine(y, H, inv, w, valid, T, k, S, co, st));
  } else {
    moe::GroupedGemmFp8Args fa;
    memset(&fa, 0, sizeof(fa));
    fa.a_routed = wts->w_gate_up;
    fa.a_shared = S ? wts->ws_gate_up : nullptr;
    fa.sa_routed = wts->s_gate_up;
    fa.sa_shared = S ? wts->ss_gate_up : nullptr;
    fa.b = at<uint8_t>(workspace, plan->off_xp);
    fa.sb = at<float>(workspace, plan->off_sx);
    fa.d = at<uint8_t>(workspace, plan->off_h);
    fa.sd = at<float>(workspace, plan->off_sh);
    fa.group_offsets = goff;
    fa.E = E;
    fa.e_base = eb;
    fa.n_local = ee - eb;
    fa.G = G;
    fa.K_routed = H;
    fa.K_shared = H;
    fa.K_ld = H;
    fa.rows_per_expert = 2 * I;
    fa.feat_routed = I;
    fa.feat_shared = S ? Is : 0;
    fa.up_routed = I;
    fa.up_shared = Is;
    fa.ldd = plan->imax;
    fa.R_cap = R_cap;
    fa.gated = true;
    fa.status = status;
    fa.timeout_bit = MOE_DEV_WAIT_TIMEOUT_GATE_UP;
    fa.wait_limit_ns = plan->wait_limit_ns;
    fa.num_ctas = plan->num_sms;
    s = check_launch(moe::launch_grouped_gemm_fp8(fa, st));
    if (s != MOE_OK) return s;
    record(dbg, 5, st);

    auto* y16 = at<__nv_bfloat16>(workspace, plan->off_y);
    fa.a_routed = wts->w_down;
    fa.a_shared = S ? wts->ws_down : nullptr;
    fa.sa_routed = wts->s_down;
    fa.sa_shared = S ? wts->ss_down : nullptr;
    fa.b = at<uint8_t>(workspace, plan->off_h);
    fa.sb = at<float>(workspace, plan->off_sh);
    fa.d = y16;
    fa.sd = nullptr;
    fa.K_routed = I;
    fa.K_shared = S ? Is : 0;
    fa.K_ld = plan->imax;
    fa.rows_per_expert = H;
    fa.feat_routed = H;
    fa.feat_shared = S ? H : 0;
    fa.up_routed = 0;
    fa.up_shared = 0;
    fa.ldd = H;
    fa.gated = false;
    fa.timeout_bit = MOE_DEV_WAIT_TIMEOUT_DOWN;
    if (send != nullptr) {
      fa.send = *send;
      fa.send.perm = perm;
      fa.send.row_token = rowtok;
      fa.send.done = at<unsigned int>(workspace, plan->off_done);
      if (cudaMemsetAsync(fa.send.done, 0, sizeof(unsigned int) * G, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
    s = check_launch(moe::launch_grouped_gemm_fp8(fa, st));
    if (s != MOE_OK) return s;
    record(dbg, 6, st);

    if (send == nullptr)
      s = check_launch(moe::launch_combine_bf16y(y16, H, inv, w, valid, T, k, S, co, st));
  }
  if (s != MOE_OK) return s;
  record(dbg, 7, st);

  if (dbg != nullptr) {
    const auto d2d = cudaMemcpyDeviceToDevice;
    if (dbg->logits && cudaMemcpyAsync(dbg->logits, logits, sizeof(float) * T * E, d2d, st))
      return MOE_ERR_CUDA;
    if (dbg->topk_ids && cudaMemcpyAsync(dbg->topk_ids, ids, sizeof(int) * T * k, d2d, st))
      return MOE_ERR_CUDA;
    if (dbg->topk_w && cudaMemcpyAsync(dbg->topk_w, w, sizeof(float) * T * k, d2d, st))
      return MOE_ERR_CUDA;
    if (dbg->perm && cudaMemcpyAsync(dbg->perm, perm, sizeof(int) * T * k, d2d, st))
      return MOE_ERR_CUDA;
    if (dbg->offsets && cudaMemcpyAsync(dbg->offsets, goff, sizeof(int) * (E + 1), d2d, st))
      return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

MOE_EXPORT moe_status moe_forward(moe_plan_t plan, const moe_weights* wts, const void* hidden,
                                  const uint8_t* valid, int T, int k, void* out, void* workspace,
                                  size_t ws_bytes, void* stream, moe_debug* dbg) {
  if (plan == nullptr || out == nullptr || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  moe::CombineOut co;
  memset(&co, 0, sizeof(co));
  co.bf16 = static_cast<__nv_bfloat16*>(out);
  return forward_impl(plan, wts, hidden, valid, T, k, co, 0, plan->cfg.num_experts, workspace,
                      ws_bytes, stream, dbg);
}

MOE_EXPORT moe_status moe_forward_scatter_experts(moe_plan_t plan, const moe_weights* wts,
                                                  const void* hidden, const uint8_t* valid, int T,
                                                  int k, float* const* dst, int n_dst,
                                                  int rows_per_rank, int slot, int expert_begin,
                                                  int expert_end, void* workspace,
                                                  size_t ws_bytes, void* stream, moe_debug* dbg) {
  if (plan == nullptr || expert_begin < 0 || expert_end <= expert_begin ||
      expert_end > plan->cfg.num_experts)
    return MOE_ERR_INVALID_ARG;
  if (dst == nullptr || n_dst < 1 || n_dst > moe::kMaxTpRanks || rows_per_rank < 1 ||
      (long long)n_dst * rows_per_rank != T || slot < 0 || slot >= n_dst)
    return MOE_ERR_INVALID_ARG;
  moe::CombineOut co;
  memset(&co, 0, sizeof(co));
  for (int r = 0; r < n_dst; ++r) {
    if (dst[r] == nullptr || !aligned16(dst[r])) return MOE_ERR_INVALID_ARG;
    co.dst[r] = dst[r];
  }
  co.rows_per_rank = rows_per_rank;
  co.slot = slot;
  return forward_impl(plan, wts, hidden, valid, T, k, co, expert_begin, expert_end, workspace,
                      ws_bytes, stream, dbg);
}

MOE_EXPORT moe_status moe_forward_scatter(moe_plan_t plan, const moe_weights* wts,
                                          const void* hidden, const uint8_t* valid, int T, int k,
                                          float* const* dst, int n_dst, int rows_per_rank,
                                          int slot, void* workspace, size_t ws_bytes,
                                          void* stream, moe_debug* dbg) {
  if (plan == nullptr) return MOE_ERR_INVALID_ARG;
  return moe_forward_scatter_experts(plan, wts, hidden, valid, T, k, dst, n_dst, rows_per_rank,
                                     slot, 0, plan->cfg.num_experts, workspace, ws_bytes, stream,
                                     dbg);
}

MOE_EXPORT moe_status moe_reduce_partials(const float* slots, int n_slots, int rows, int H,
                                          const uint8_t* valid, void* out, void* stream) {
  if (slots == nullptr || out == nullptr || n_slots < 1 || n_slots > moe::kMaxTpRanks ||
      rows < 0 || H <= 0 || H % 8 != 0 || !aligned16(slots) || !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  return check_launch(moe::launch_reduce_slots(slots, n_slots, rows, H, valid,
                                               static_cast<__nv_bfloat16*>(out),
                                               static_cast<cudaStream_t>(stream)));
}

MOE_EXPORT moe_status moe_forward_scatter_pairs(moe_plan_t plan, const moe_weights* wts,
                                                const void* hidden, const uint8_t* valid, int T,
                                                int k, float* const* dst, int n_dst,
                                                int rows_per_rank, int shared_slot,
                                                int expert_begin, int expert_end, int send_ctas,
                                                void* workspace, size_t ws_bytes, void* stream,
                                                moe_debug* dbg) {
  if (plan == nullptr || expert_begin < 0 || expert_end <= expert_begin ||
      expert_end > plan->cfg.num_experts || send_ctas < 1)
    return MOE_ERR_INVALID_ARG;
  if (dst == nullptr || n_dst < 1 || n_dst > moe::kMaxTpRanks || rows_per_rank < 1 ||
      (long long)n_dst * rows_per_rank != T)
    return MOE_ERR_INVALID_ARG;
  if (plan->cfg.num_shared && shared_slot < k) return MOE_ERR_INVALID_ARG;
  moe::SendArgs sa;
  memset(&sa, 0, sizeof(sa));
  for (int r = 0; r < n_dst; ++r) {
    if (dst[r] == nullptr || !aligned16(dst[r])) return MOE_ERR_INVALID_ARG;
    sa.dst[r] = dst[r];
  }
  sa.rows_per_rank = rows_per_rank;
  sa.k = k;
  sa.shared_slot = shared_slot;
  sa.n_send = send_ctas;
  sa.timeout_bit = MOE_DEV_WAIT_TIMEOUT_SEND;
  moe::CombineOut co;
  memset(&co, 0, sizeof(co));
  return forward_impl(plan, wts, hidden, valid, T, k, co, expert_begin, expert_end, workspace,
                      ws_bytes, stream, dbg, &sa);
}

MOE_EXPORT moe_status moe_reduce_pairs(const float* slab, int k, int n_extra, int rows, int H,
                                       const float* w, const uint8_t* valid, void* out,
                                       void* stream) {
  if (slab == nullptr || w == nullptr || out == nullptr || k < 1 || k > moe::kMaxTopK ||
      n_extra < 0 || n_extra > moe::kMaxTpRanks || rows < 0 || H <= 0 || H % 8 != 0 ||
      !aligned16(slab) || !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  return check_launch(moe::launch_reduce_pairs(slab, k, n_extra, rows, H, w, valid,
                                               static_cast<__nv_bfloat16*>(out),
                                               static_cast<cudaStream_t>(stream)));
}

MOE_EXPORT moe_status moe_route_from_logits(moe_plan_t plan, const float* logits,
                                            const uint8_t* valid, int T, int k, int* topk_ids,
                                            float* topk_w, int* perm, int* offsets,
                                            void* workspace, size_t ws_bytes, void* stream) {
  moe_status s = check_common(plan, T, k, workspace, ws_bytes);
  if (s != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  if (logits == nullptr || topk_ids == nullptr || topk_w == nullptr || perm == nullptr ||
      offsets == nullptr)
    return MOE_ERR_INVALID_ARG;
  s = ensure_device(plan);
  if (s != MOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const moe_config& c = plan->cfg;
  const int E = c.num_experts, S = c.num_shared;
  unsigned int* status = at<unsigned int>(workspace, plan->off_status);
  int* goff = at<int>(workspace, plan->off_goff);
  if (cudaMemsetAsync(status, 0, sizeof(unsigned int), st) != cudaSuccess) return MOE_ERR_CUDA;
  s = check_launch(moe::launch_topk(logits, 1, nullptr, valid, T, E, k, c.renormalize,
                                    at<float>(workspace, plan->off_logits), topk_ids, topk_w, st));
  if (s != MOE_OK) return s;
  s = check_launch(moe::launch_route(topk_ids, valid, T, E, k, S, 0, E, goff, perm,
                                     at<int>(workspace, plan->off_inv),
                                     at<int>(workspace, plan->off_rowtok), status,
                                     at<int>(workspace, plan->off_rscratch), st));
  if (s != MOE_OK) return s;
  if (cudaMemcpyAsync(offsets, goff, sizeof(int) * (E + 1), cudaMemcpyDeviceToDevice, st) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

MOE_EXPORT moe_status moe_check_device_status(moe_plan_t plan, void* workspace, void* stream,
                                              uint32_t* bits) {
  if (plan == nullptr || workspace == nullptr) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned int* status = at<unsigned int>(workspace, plan->off_status);
  unsigned int v = 0;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpy(&v, status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (v != 0 && cudaMemset(status, 0, sizeof(v)) != cudaSuccess) return MOE_ERR_CUDA;
  if (bits != nullptr) *bits = v;
  return v == 0 ? MOE_OK : MOE_ERR_DEVICE;
}

MOE_EXPORT moe_status moe_get_workspace_views(moe_plan_t plan, void* workspace,
                                              moe_workspace_views* v) {
  if (plan == nullptr || workspace == nullptr || v == nullptr) return MOE_ERR_INVALID_ARG;
  v->row_token = at<int>(workspace, plan->off_rowtok);
  v->x_perm = at<void>(workspace, plan->off_xp);
  v->h = at<void>(workspace, plan->off_h);
  v->y = at<void>(workspace, plan->off_y);
  v->group_offsets = at<int>(workspace, plan->off_goff);
  v->h_stride = plan->imax;
  const bool fp8 = plan->cfg.wtype == MOE_W_FP8_E4M3_B128;
  v->x_scale = fp8 ? at<float>(workspace, plan->off_sx) : nullptr;
  v->h_scale = fp8 ? at<float>(workspace, plan->off_sh) : nullptr;
  return MOE_OK;
}

// ------------------------------------------------------------------ pipeline
// Host-to-host forwards: uploads and downloads on two copy streams, forwards on
// a compute stream, one slot of device buffers per batch in flight.

constexpr int kMaxPipelineDepth = 8;

struct moe_pipeline_s {
  moe_plan_t plan = nullptr;
  moe_weights wts;
  int k = 0, rows = 0, depth = 0;
  bool graph = false;
  uint8_t* slots = nullptr;
  size_t stride = 0, off_valid = 0, off_out = 0;
  void* workspace = nullptr;
  size_t ws_bytes = 0;
  cudaStream_t up = nullptr, compute = nullptr, down = nullptr;
  cudaEvent_t loaded[kMaxPipelineDepth] = {};
  cudaEvent_t computed[kMaxPipelineDepth] = {};
  cudaEvent_t drained[kMaxPipelineDepth] = {};
  cudaGraphExec_t exec[kMaxPipelineDepth] = {};
  bool used[kMaxPipelineDepth] = {};
  long long count = 0;
};

namespace {

// per slot: x bf16 [rows, H], valid uint8 [rows], out bf16 [rows, H], each 256-byte aligned
void pipeline_layout(const moe_plan_s* p, int rows, size_t* off_valid, size_t* off_out,
                     size_t* stride) {
  const size_t xb = align_up((size_t)rows * p->cfg.hidden * 2);
  *off_valid = xb;
  *off_out = xb + align_up((size_t)rows);
  *stride = *off_out + xb;
}

void pipeline_release(moe_pipeline_s* q) {
  for (int s = 0; s < kMaxPipelineDepth; ++s) {
    if (q->exec[s] != nullptr) cudaGraphExecDestroy(q->exec[s]);
    if (q->loaded[s] != nullptr) cudaEventDestroy(q->loaded[s]);
    if (q->computed[s] != nullptr) cudaEventDestroy(q->computed[s]);
    if (q->drained[s] != nullptr) cudaEventDestroy(q->drained[s]);
  }
  if (q->up != nullptr) cudaStreamDestroy(q->up);
  if (q->compute != nullptr) cudaStreamDestroy(q->compute);
  if (q->down != nullptr) cudaStreamDestroy(q->down);
  delete q;
}

moe_status cuda_status(cudaError_t e) { return check_launch(e); }

// slot s's forward on the compute stream (the moe_forward launch sequence)
moe_status pipeline_forward(moe_pipeline_s* q, int s) {
  uint8_t* base = q->slots + (size_t)s * q->stride;
  moe::CombineOut co;
  memset(&co, 0, sizeof(co));
  co.bf16 = reinterpret_cast<__nv_bfloat16*>(base + q->off_out);
  return forward_impl(q->plan, &q->wts, base, base + q->off_valid, q->rows, q->k, co, 0,
                      q->plan->cfg.num_experts, q->workspace, q->ws_bytes, q->compute, nullptr);
}

}  // namespace

MOE_EXPORT moe_status moe_pipeline_slot_bytes(moe_plan_t plan, int rows, int depth,
                                              size_t* bytes) {
  if (plan == nullptr || bytes == nullptr || rows < 1 || rows > plan->cfg.max_tokens ||
      depth < 1 || depth > kMaxPipelineDepth)
    return MOE_ERR_INVALID_ARG;
  size_t ov = 0, oo = 0, stride = 0;
  pipeline_layout(plan, rows, &ov, &oo, &stride);
  *bytes = stride * (size_t)depth;
  return MOE_OK;
}

MOE_EXPORT moe_status moe_pipeline_create(moe_plan_t plan, const moe_weights* wts, int k,
                                          int rows, int depth, int use_graph, void* slots,
                                          size_t slots_bytes, void* workspace, size_t ws_bytes,
                                          moe_pipeline_t* pipeline) {
  if (pipeline == nullptr) return MOE_ERR_INVALID_ARG;
  *pipeline = nullptr;
  if (wts == nullptr) return MOE_ERR_INVALID_ARG;
  size_t need = 0;
  moe_status st = moe_pipeline_slot_bytes(plan, rows, depth, &need);
  if (st != MOE_OK) return st;
  if (k < 1 || k > plan->cfg.top_k_max) return MOE_ERR_INVALID_ARG;
  if (slots == nullptr || (reinterpret_cast<uintptr_t>(slots) & (kAlign - 1)) != 0)
    return MOE_ERR_INVALID_ARG;
  if (slots_bytes < need) return MOE_ERR_WORKSPACE;
  st = check_common(plan, rows, k, workspace, ws_bytes);
  if (st != MOE_OK) return st;

  moe_pipeline_s* q = new (std::nothrow) moe_pipeline_s;
  if (q == nullptr) return MOE_ERR_INVALID_ARG;
  q->plan = plan;
  q->wts = *wts;
  q->k = k;
  q->rows = rows;
  q->depth = depth;
  q->graph = use_graph != 0;
  q->slots = static_cast<uint8_t*>(slots);
  pipeline_layout(plan, rows, &q->off_valid, &q->off_out, &q->stride);
  q->workspace = workspace;
  q->ws_bytes = ws_bytes;

  // the weights and buffers the caller prepared on any stream are ready after this
  st = cuda_status(cudaDeviceSynchronize());
  if (st == MOE_OK) st = cuda_status(cudaStreamCreateWithFlags(&q->up, cudaStreamNonBlocking));
  if (st == MOE_OK)
    st = cuda_status(cudaStreamCreateWithFlags(&q->compute, cudaStreamNonBlocking));
  if (st == MOE_OK) st = cuda_status(cudaStreamCreateWithFlags(&q->down, cudaStreamNonBlocking));
  for (int s = 0; s < depth && st == MOE_OK; ++s) {
    st = cuda_status(cudaEventCreateWithFlags(&q->loaded[s], cudaEventDisableTiming));
    if (st == MOE_OK)
      st = cuda_status(cudaEventCreateWithFlags(&q->computed[s], cudaEventDisableTiming));
    if (st == MOE_OK)
      st = cuda_status(cudaEventCreateWithFlags(&q->drained[s], cudaEventDisableTiming));
  }
  // all-padding batches in every slot; the first forward of each runs outside any
  // capture (kernel attributes are set on first use)
  if (st == MOE_OK) st = cuda_status(cudaMemsetAsync(slots, 0, need, q->compute));
  for (int s = 0; s < depth && st == MOE_OK; ++s) st = pipeline_forward(q, s);
  if (st == MOE_OK) st = cuda_status(cudaStreamSynchronize(q->compute));
  for (int s = 0; s < depth && st == MOE_OK && q->graph; ++s) {
    st = cuda_status(cudaStreamBeginCapture(q->compute, cudaStreamCaptureModeThreadLocal));
    if (st != MOE_OK) break;
    const moe_status fs = pipeline_forward(q, s);
    cudaGraph_t g = nullptr;
    const cudaError_t ce = cudaStreamEndCapture(q->compute, &g);
    if (fs != MOE_OK || ce != cudaSuccess || g == nullptr) {
      if (g != nullptr) cudaGraphDestroy(g);
      st = fs != MOE_OK ? fs : cuda_status(ce != cudaSuccess ? ce : cudaErrorUnknown);
      break;
    }
    st = cuda_status(cudaGraphInstantiate(&q->exec[s], g, 0));
    cudaGraphDestroy(g);
  }
  if (st == MOE_OK) st = cuda_status(cudaStreamSynchronize(q->compute));
  if (st != MOE_OK) {
    pipeline_release(q);
    return st;
  }
  *pipeline = q;
  return MOE_OK;
}

MOE_EXPORT moe_status moe_pipeline_submit(moe_pipeline_t q, const void* hidden_host,
                                          const uint8_t* valid_host, void* out_host) {
  if (q == nullptr || hidden_host == nullptr || out_host == nullptr) return MOE_ERR_INVALID_ARG;
  const int s = (int)(q->count % q->depth);
  uint8_t* base = q->slots + (size_t)s * q->stride;
  const size_t xb = (size_t)q->rows * q->plan->cfg.hidden * 2;
  // refill a slot only after its previous output has been downloaded (which
  // itself followed that forward, the last reader of the slot's inputs)
  moe_status st = MOE_OK;
  if (q->used[s]) st = cuda_status(cudaStreamWaitEvent(q->up, q->drained[s], 0));
  if (st == MOE_OK)
    st = cuda_status(cudaMemcpyAsync(base, hidden_host, xb, cudaMemcpyHostToDevice, q->up));
  if (st == MOE_OK)
    st = cuda_status(valid_host != nullptr
                         ? cudaMemcpyAsync(base + q->off_valid, valid_host, (size_t)q->rows,
                                           cudaMemcpyHostToDevice, q->up)
                         : cudaMemsetAsync(base + q->off_valid, 1, (size_t)q->rows, q->up));
  if (st == MOE_OK) st = cuda_status(cudaEventRecord(q->loaded[s], q->up));
  if (st == MOE_OK) st = cuda_status(cudaStreamWaitEvent(q->compute, q->loaded[s], 0));
  if (st == MOE_OK)
    st = q->graph ? cuda_status(cudaGraphLaunch(q->exec[s], q->compute)) : pipeline_forward(q, s);
  if (st == MOE_OK) st = cuda_status(cudaEventRecord(q->computed[s], q->compute));
  if (st == MOE_OK) st = cuda_status(cudaStreamWaitEvent(q->down, q->computed[s], 0));
  if (st == MOE_OK)
    st = cuda_status(
        cudaMemcpyAsync(out_host, base + q->off_out, xb, cudaMemcpyDeviceToHost, q->down));
  if (st == MOE_OK) st = cuda_status(cudaEventRecord(q->drained[s], q->down));
  if (st != MOE_OK) return st;
  q->used[s] = true;
  ++q->count;
  return MOE_OK;
}

MOE_EXPORT moe_status moe_pipeline_synchronize(moe_pipeline_t q) {
  if (q == nullptr) return MOE_ERR_INVALID_ARG;
  return cuda_status(cudaStreamSynchronize(q->down));
}

MOE_EXPORT moe_status moe_pipeline_streams(moe_pipeline_t q, void** upload, void** compute,
                                           void** download) {
  if (q == nullptr) return MOE_ERR_INVALID_ARG;
  if (upload != nullptr) *upload = q->up;
  if (compute != nullptr) *compute = q->compute;
  if (download != nullptr) *download = q->down;
  return MOE_OK;
}

MOE_EXPORT void moe_pipeline_destroy(moe_pipeline_t q) {
  if (q == nullptr) return;
  cudaStreamSynchronize(q->up);
  cudaStreamSynchronize(q->compute);
  cudaStreamSynchronize(q->down);
  pipeline_release(q);
}

namespace moe {
const moe_config* plan_config(const moe_plan_s* plan) { return &plan->cfg; }
}  // namespace moe
