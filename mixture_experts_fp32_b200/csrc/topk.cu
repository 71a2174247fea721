// Top-k expert selection and routing weights from fp32 logits (Step3 推論最適化
// (MI308X vs H20), §背景: each token keeps 3 of 48 experts).
//
// topk_kernel: one warp per token.  It adds the router's split-K partial sums
// in split order (plus the per-expert bias), keeps the logits (when logits_out
// is not null), and runs k
// rounds of a warp arg-max under the order (logit descending, expert
// ascending); the weights are the softmax of the selected logits
// (renormalised) or their full-softmax probabilities.
#include "moe_internal.cuh"

namespace moe {
namespace {

// (v, e) is better than (bv, be) under: larger logit first, then lower index.
__device__ __forceinline__ bool better(float v, int e, float bv, int be) {
  return v > bv || (v == bv && e < be);
}

// NB: splits whose loads are issued together (4 for a few splits, where fewer
// registers keep more warps resident; 8 when the router split K many ways)
template <int NB>
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
    if (logits_out != nullptr)
      for (int e = lane; e < E; e += 32) logits_out[(size_t)t * E + e] = 0.f;
    if (lane < k) {
      ids[(size_t)t * k + lane] = -1;
      w[(size_t)t * k + lane] = 0.f;
    }
    return;
  }

  // the splits are added in order, each element's sum starting from 0; the loads of
  // NB splits for all of the lane's experts go out together (one round trip per NB
  // splits, not one per split and expert)
  float v[8];
  uint32_t avail = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[i] = 0.f;
    if (i < per_lane && lane + 32 * i < E) avail |= 1u << i;
  }
  for (int sp0 = 0; sp0 < splits; sp0 += NB) {
    float pv[NB][8];                      // NB splits' loads before any of their adds
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const float* prow = partial + ((size_t)(sp0 + b) * T + t) * E + lane;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        pv[b][i] = (sp0 + b < splits && ((avail >> i) & 1u)) ? prow[32 * i] : 0.f;
    }
#pragma unroll
    for (int b = 0; b < NB; ++b)
      if (sp0 + b < splits) {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] += pv[b][i];
      }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    if ((avail >> i) & 1u) {
      if (bias != nullptr) v[i] += bias[e];
      if (logits_out != nullptr) logits_out[(size_t)t * E + e] = v[i];
    } else {
      v[i] = 0.f;
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

cudaError_t launch_topk(const float* partial, int splits, const float* bias, const uint8_t* valid,
                        int T, int E, int k, int renorm, float* logits_out, int* ids, float* w,
                        cudaStream_t st) {
  const int warps = 8;
  const int grid = (T + warps - 1) / warps;
  if (splits > 4)
    topk_kernel<8><<<grid, warps * 32, 0, st>>>(partial, splits, bias, valid, T, E, k, renorm,
                                                logits_out, ids, w);
  else
    topk_kernel<4><<<grid, warps * 32, 0, st>>>(partial, splits, bias, valid, T, E, k, renorm,
                                                logits_out, ids, w);
  return cudaGetLastError();
}

}  // namespace moe
