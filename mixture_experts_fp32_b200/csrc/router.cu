// Router: logits l[t,e] = sum_h x[t,h] Wr[e,h] (+ b[e]) in fp32, then the
// top-k selection and the routing weights (Step3 推論最適化 (MI308X vs H20),
// §背景: each token selects 3 of 48 experts).
//
// router_logits_kernel: a tiled fp32 SIMT GEMM (32 tokens x 32 experts per
//   block, K staged through shared memory), split along H so that decode-sized
//   batches still fill the GPU.  Each split writes its own partial sums; the
//   top-k kernel adds them in split order, so the result is deterministic.
//   Tiles whose 32 rows are all padding are skipped.
// topk_kernel: one warp per token.  Each lane holds up to 8 logits; k rounds
//   of a warp arg-max under the order (logit descending, expert ascending)
//   select the experts; the weights are the softmax of the selected logits
//   (renormalised) or their full-softmax probabilities.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int RT = 32;   // tokens per tile
constexpr int RE = 32;   // experts per tile
constexpr int RK = 32;   // K elements per shared-memory stage

__global__ void __launch_bounds__(256) router_logits_kernel(const __nv_bfloat16* __restrict__ x,
                                                            const uint8_t* __restrict__ valid,
                                                            int T, int H,
                                                            const float* __restrict__ Wr, int E,
                                                            float* __restrict__ partial,
                                                            int kchunk) {
  __shared__ float xs[RK][RT + 1];
  __shared__ float ws[RK][RE + 1];
  __shared__ int any_valid;
  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * RT, e0 = blockIdx.y * RE, split = blockIdx.z;
  const int kbeg = split * kchunk;
  const int kend = min(H, kbeg + kchunk);

  if (tid == 0) any_valid = 0;
  __syncthreads();
  if (tid < RT && t0 + tid < T && (valid == nullptr || valid[t0 + tid])) any_valid = 1;
  __syncthreads();
  if (!any_valid || kbeg >= kend) return;

  const int ty = tid / 16, tx = tid % 16;   // 2 tokens x 2 experts per thread
  float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};

  const int lr = tid / 8, lc = (tid % 8) * 4;   // loader: row lr, 4 columns from lc
  const int lt = t0 + lr, le = e0 + lr;
  const bool x_ok = lt < T && (valid == nullptr || valid[lt]);
  const bool w_ok = le < E;

  for (int kc = kbeg; kc < kend; kc += RK) {
    float xv[4] = {0.f, 0.f, 0.f, 0.f};
    if (x_ok) {
      const uint2 raw = *reinterpret_cast<const uint2*>(x + (size_t)lt * H + kc + lc);
      const __nv_bfloat162 p0 = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
      const __nv_bfloat162 p1 = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
      xv[0] = __low2float(p0); xv[1] = __high2float(p0);
      xv[2] = __low2float(p1); xv[3] = __high2float(p1);
    }
    float4 wv = make_float4(0.f, 0.f, 0.f, 0.f);
    if (w_ok) wv = *reinterpret_cast<const float4*>(Wr + (size_t)le * H + kc + lc);
    xs[lc + 0][lr] = xv[0]; xs[lc + 1][lr] = xv[1]; xs[lc + 2][lr] = xv[2]; xs[lc + 3][lr] = xv[3];
    ws[lc + 0][lr] = wv.x; ws[lc + 1][lr] = wv.y; ws[lc + 2][lr] = wv.z; ws[lc + 3][lr] = wv.w;
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < RK; ++kk) {
      const float a0 = xs[kk][2 * ty], a1 = xs[kk][2 * ty + 1];
      const float b0 = ws[kk][2 * tx], b1 = ws[kk][2 * tx + 1];
      acc[0][0] = fmaf(a0, b0, acc[0][0]);
      acc[0][1] = fmaf(a0, b1, acc[0][1]);
      acc[1][0] = fmaf(a1, b0, acc[1][0]);
      acc[1][1] = fmaf(a1, b1, acc[1][1]);
    }
    __syncthreads();
  }
  float* out = partial + (size_t)split * T * E;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int t = t0 + 2 * ty + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int e = e0 + 2 * tx + j;
      if (e < E) out[(size_t)t * E + e] = acc[i][j];
    }
  }
}

// (v, e) is better than (bv, be) under: larger logit first, then lower index.
__device__ __forceinline__ bool better(float v, int e, float bv, int be) {
  return v > bv || (v == bv && e < be);
}

__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ partial, int splits,
                                                   const float* __restrict__ bias,
                                                   const uint8_t* __restrict__ valid, int T, int E,
                                                   int k, int renorm,
                                                   float* __restrict__ logits_out,
                                                   int* __restrict__ ids, float* __restrict__ w) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (t >= T) return;
  constexpr int kNone = 0x7fffffff;
  const int per_lane = (E + 31) / 32;   // <= 8

  if (valid != nullptr && !valid[t]) {
    for (int e = lane; e < E; e += 32) logits_out[(size_t)t * E + e] = 0.f;
    if (lane < k) {
      ids[(size_t)t * k + lane] = -1;
      w[(size_t)t * k + lane] = 0.f;
    }
    return;
  }

  float v[8];
  uint32_t avail = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[i] = 0.f;
    const int e = lane + 32 * i;
    if (i < per_lane && e < E) {
      float s = 0.f;
      for (int sp = 0; sp < splits; ++sp) s += partial[((size_t)sp * T + t) * E + e];
      if (bias != nullptr) s += bias[e];
      v[i] = s;
      logits_out[(size_t)t * E + e] = s;
      avail |= 1u << i;
    }
  }

  int sel_e[kMaxTopK];
  float sel_v[kMaxTopK];
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    sel_e[j] = 0;
    sel_v[j] = 0.f;
    if (j >= k) continue;
    float bv = 0.f;
    int be = kNone;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if ((avail >> i) & 1u) {
        const int e = lane + 32 * i;
        if (be == kNone || better(v[i], e, bv, be)) { bv = v[i]; be = e; }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (oe != kNone && (be == kNone || better(ov, oe, bv, be))) { bv = ov; be = oe; }
    }
    sel_e[j] = be;
    sel_v[j] = bv;
    if ((be & 31) == lane) avail &= ~(1u << (be >> 5));
  }

  const float m = sel_v[0];
  float z = 0.f;
  if (renorm) {
    for (int j = 0; j < k; ++j) z += expf(sel_v[j] - m);
  } else {
    float part = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      if (i < per_lane && e < E) part += expf(v[i] - m);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    z = part;
  }
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    if (j < k && lane == j) {
      ids[(size_t)t * k + j] = sel_e[j];
      w[(size_t)t * k + j] = expf(sel_v[j] - m) / z;
    }
  }
}

}  // namespace

void router_split_plan(int T, int E, int H, int num_sms, int* splits_out, int* kchunk_out) {
  const int tiles = ((T + RT - 1) / RT) * ((E + RE - 1) / RE);
  int splits = (2 * num_sms + tiles - 1) / tiles;
  if (splits < 1) splits = 1;
  if (splits > kRouterSplitMax) splits = kRouterSplitMax;
  if (splits > H / RK) splits = H / RK;
  // a whole number of RK stages per split; every split gets at least one
  int kchunk = (H + splits - 1) / splits;
  kchunk = (kchunk + RK - 1) / RK * RK;
  *kchunk_out = kchunk;
  *splits_out = (H + kchunk - 1) / kchunk;
}

cudaError_t launch_router_logits(const __nv_bfloat16* x, const uint8_t* valid, int T, int H,
                                 const float* Wr, int E, float* partial, int splits, int kchunk,
                                 cudaStream_t st) {
  dim3 grid((T + RT - 1) / RT, (E + RE - 1) / RE, splits);
  router_logits_kernel<<<grid, 256, 0, st>>>(x, valid, T, H, Wr, E, partial, kchunk);
  return cudaGetLastError();
}

cudaError_t launch_topk(const float* partial, int splits, const float* bias, const uint8_t* valid,
                        int T, int E, int k, int renorm, float* logits_out, int* ids, float* w,
                        cudaStream_t st) {
  const int warps = 8;
  topk_kernel<<<(T + warps - 1) / warps, warps * 32, 0, st>>>(partial, splits, bias, valid, T, E,
                                                              k, renorm, logits_out, ids, w);
  return cudaGetLastError();
}

}  // namespace moe
