// Token permutation (group-by-expert), row gather and the weighted combine.
//
// route_kernel: one block of 1024 threads builds, deterministically and with
//   no global atomics, the per-expert offsets, the permutation perm (pairs
//   t*k+j grouped by expert, ascending t inside an expert), its inverse, and
//   the row -> token map that the GEMMs use.  Rows are grouped as: routed
//   experts 0..E-1, then (S = 1) the shared expert, which takes every valid
//   token in ascending order.  Padding rows are skipped.  Tokens are processed
//   in chunks of 1024; inside a chunk, a shared-memory bitmap per expert (one
//   bit per token) gives each pair its rank by population counts.
// gather_rows_kernel: x_perm[r] = x[row_token[r]] with 16-byte vectors.
// combine_kernel: out[t] = bf16( sum_j w[t,j] y[inv[t,j]] + y[inv[t,k]] ),
//   y in fp32, summed in fp32 in ascending j, shared expert last; padding rows get +0.0
//   (the combine phase, [SGLang] MoE 모델을 위한 Single Batch Overlap 기법,
//   §들어가며; the fused shared expert, Step3 推論最適化 (MI308X vs H20),
//   §最適化技術).
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kChunk = 1024;

__device__ __forceinline__ void set_bits(uint32_t (*bits)[32], const int* ids, const uint8_t* valid,
                                         int T, int E, int k, int t, int warp, int lane,
                                         unsigned int* status) {
  if (t < T && (valid == nullptr || valid[t])) {
    for (int j = 0; j < k; ++j) {
      const int e = ids[(size_t)t * k + j];
      if (e < 0 || e >= E) {
        atomicOr(status, MOE_DEV_BAD_EXPERT_ID);
        continue;
      }
      atomicOr(&bits[e][warp], 1u << lane);
    }
  }
}

__global__ void __launch_bounds__(1024, 1) route_kernel(const int* __restrict__ ids,
                                                        const uint8_t* __restrict__ valid, int T,
                                                        int E, int k, int S,
                                                        int* __restrict__ group_offsets,
                                                        int* __restrict__ perm,
                                                        int* __restrict__ inv,
                                                        int* __restrict__ row_token,
                                                        unsigned int* status) {
  __shared__ uint32_t bits[kMaxExperts][32];
  __shared__ int run[kMaxExperts];
  __shared__ int wvalid[32];
  __shared__ int s_valid_total, s_vrun;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int nchunks = (T + kChunk - 1) / kChunk;

  for (int e = tid; e < E; e += blockDim.x) run[e] = 0;
  if (tid == 0) { s_valid_total = 0; s_vrun = 0; }
  __syncthreads();

  // pass 1: per-expert pair counts and the valid-token count
  for (int c = 0; c < nchunks; ++c) {
    for (int i = tid; i < E * 32; i += blockDim.x) bits[i >> 5][i & 31] = 0u;
    __syncthreads();
    const int t = c * kChunk + tid;
    set_bits(bits, ids, valid, T, E, k, t, warp, lane, status);
    const bool ok = t < T && (valid == nullptr || valid[t]);
    const uint32_t vb = __ballot_sync(0xffffffffu, ok);
    if (lane == 0) wvalid[warp] = __popc(vb);
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
      int s = 0;
      for (int w = 0; w < 32; ++w) s += __popc(bits[e][w]);
      run[e] += s;
    }
    if (tid == 0) {
      int s = 0;
      for (int w = 0; w < 32; ++w) s += wvalid[w];
      s_valid_total += s;
    }
    __syncthreads();
  }

  // exclusive scan of the counts: group offsets (routed experts, then shared)
  if (tid == 0) {
    int acc = 0;
    for (int e = 0; e < E; ++e) {
      const int c = run[e];
      group_offsets[e] = acc;
      run[e] = acc;
      acc += c;
    }
    group_offsets[E] = acc;
    if (S) group_offsets[E + 1] = acc + s_valid_total;
  }
  __syncthreads();
  const int routed_rows = group_offsets[E];
  const int ks = k + S;

  // pass 2: ranks, permutation, inverse, row -> token
  for (int c = 0; c < nchunks; ++c) {
    for (int i = tid; i < E * 32; i += blockDim.x) bits[i >> 5][i & 31] = 0u;
    __syncthreads();
    const int t = c * kChunk + tid;
    set_bits(bits, ids, valid, T, E, k, t, warp, lane, status);
    const bool ok = t < T && (valid == nullptr || valid[t]);
    const uint32_t vb = __ballot_sync(0xffffffffu, ok);
    if (lane == 0) wvalid[warp] = __popc(vb);
    __syncthreads();
    if (t < T) {
      if (ok) {
        for (int j = 0; j < k; ++j) {
          const int e = ids[(size_t)t * k + j];
          if (e < 0 || e >= E) {
            inv[(size_t)t * ks + j] = -1;
            continue;
          }
          int r = run[e];
          for (int w = 0; w < warp; ++w) r += __popc(bits[e][w]);
          r += __popc(bits[e][warp] & lt_mask);
          perm[r] = t * k + j;
          inv[(size_t)t * ks + j] = r;
          row_token[r] = t;
        }
        if (S) {
          int vr = s_vrun + __popc(vb & lt_mask);
          for (int w = 0; w < warp; ++w) vr += wvalid[w];
          const int pos = routed_rows + vr;
          inv[(size_t)t * ks + k] = pos;
          row_token[pos] = t;
        }
      } else {
        for (int j = 0; j < ks; ++j) inv[(size_t)t * ks + j] = -1;
      }
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
      int s = 0;
      for (int w = 0; w < 32; ++w) s += __popc(bits[e][w]);
      run[e] += s;
    }
    if (tid == 0) {
      int s = 0;
      for (int w = 0; w < 32; ++w) s += wvalid[w];
      s_vrun += s;
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(256) gather_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                          int H,
                                                          const int* __restrict__ row_token,
                                                          const int* __restrict__ total_rows,
                                                          __nv_bfloat16* __restrict__ xp) {
  const int R = *total_rows;
  const int nv = H / 8;
  for (int r = blockIdx.x; r < R; r += gridDim.x) {
    const int t = row_token[r];
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
    uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)r * H);
    for (int v = threadIdx.x; v < nv; v += blockDim.x) dst[v] = src[v];
  }
}

// acc[0..7] += wgt * y[8 consecutive fp32]
__device__ __forceinline__ void acc_row(float (&acc)[8], const float* y8, float wgt) {
  const float4 a = reinterpret_cast<const float4*>(y8)[0];
  const float4 b = reinterpret_cast<const float4*>(y8)[1];
  acc[0] = fmaf(wgt, a.x, acc[0]); acc[1] = fmaf(wgt, a.y, acc[1]);
  acc[2] = fmaf(wgt, a.z, acc[2]); acc[3] = fmaf(wgt, a.w, acc[3]);
  acc[4] = fmaf(wgt, b.x, acc[4]); acc[5] = fmaf(wgt, b.y, acc[5]);
  acc[6] = fmaf(wgt, b.z, acc[6]); acc[7] = fmaf(wgt, b.w, acc[7]);
}

__device__ __forceinline__ void add_row(float (&acc)[8], const float* y8) {
  const float4 a = reinterpret_cast<const float4*>(y8)[0];
  const float4 b = reinterpret_cast<const float4*>(y8)[1];
  acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
  acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
}

__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ y, int H,
                                                      const int* __restrict__ inv,
                                                      const float* __restrict__ w,
                                                      const uint8_t* __restrict__ valid, int T,
                                                      int k, int S,
                                                      __nv_bfloat16* __restrict__ out) {
  __shared__ int rows[kMaxTopK + 1];
  __shared__ float wts[kMaxTopK];
  const int ks = k + S;
  const int nv = H / 8;
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    const bool ok = valid == nullptr || valid[t];
    if (threadIdx.x < ks) rows[threadIdx.x] = ok ? inv[(size_t)t * ks + threadIdx.x] : -1;
    if (threadIdx.x < k) wts[threadIdx.x] = ok ? w[(size_t)t * k + threadIdx.x] : 0.f;
    __syncthreads();
    uint4* dst = reinterpret_cast<uint4*>(out + (size_t)t * H);
    for (int v = threadIdx.x; v < nv; v += blockDim.x) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (ok) {
        for (int j = 0; j < k; ++j) {
          const int r = rows[j];
          if (r < 0) continue;
          acc_row(acc, y + (size_t)r * H + (size_t)v * 8, wts[j]);
        }
        if (S && rows[k] >= 0) {
          add_row(acc, y + (size_t)rows[k] * H + (size_t)v * 8);
        }
      }
      uint4 o;
      __nv_bfloat162* po = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
      for (int i = 0; i < 4; ++i) po[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
      dst[v] = o;
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_route(const int* ids, const uint8_t* valid, int T, int E, int k, int S,
                         int* group_offsets, int* perm, int* inv, int* row_token,
                         unsigned int* status, cudaStream_t st) {
  route_kernel<<<1, 1024, 0, st>>>(ids, valid, T, E, k, S, group_offsets, perm, inv, row_token,
                                   status);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const __nv_bfloat16* x, int H, const int* row_token,
                               const int* total_rows, int R_cap, __nv_bfloat16* xp, int num_sms,
                               cudaStream_t st) {
  int grid = num_sms * 8;
  if (grid > R_cap) grid = R_cap;
  if (grid < 1) grid = 1;
  gather_rows_kernel<<<grid, 256, 0, st>>>(x, H, row_token, total_rows, xp);
  return cudaGetLastError();
}

cudaError_t launch_combine(const float* y, int H, const int* inv, const float* w,
                           const uint8_t* valid, int T, int k, int S, __nv_bfloat16* out,
                           cudaStream_t st) {
  int grid = T < 148 * 16 ? T : 148 * 16;
  if (grid < 1) grid = 1;
  combine_kernel<<<grid, 256, 0, st>>>(y, H, inv, w, valid, T, k, S, out);
  return cudaGetLastError();
}

}  // namespace moe
