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
// combine_flat_kernel (fp32 y) / combine_kernel (bf16 y, a block per token):
//   out[t] = bf16( sum_j w[t,j] y[inv[t,j]] + y[inv[t,k]] ),
//   summed in fp32 in ascending j, shared expert last; padding rows get +0.0
//   (the combine phase, [SGLang] MoE 모델을 위한 Single Batch Overlap 기법,
//   §들어가며; the fused shared expert, Step3 推論最適化 (MI308X vs H20),
//   §最適化技術).  For tensor parallelism the same sum (this rank's share of the
//   intermediate dimension) is written unrounded in fp32 straight into the
//   receive slab of the rank that owns the token, possibly another GPU's memory
//   (plain stores), which is the data movement of the reduce-scatter; the owner
//   then sums its slab in rank order and rounds once (reduce_slots_kernel)
//   (TP MoE with all_gather / reduce_scatter, DP Attention and TBO for
//   DeepSeek-V4 on MI355X, introduction).
#include <cuda_fp8.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kChunk = 1024;
constexpr int kScatterSplit = 4;   // blocks that share one chunk's scatter

// Pairs routed to experts outside [eb, ee) (the experts this call computes; all of
// them, 0..E, unless a rank of an expert-parallel layer owns only a range) are left
// out of the permutation: their groups stay empty and their inverse entries are -1.
__device__ __forceinline__ void set_bits(uint32_t (*bits)[32], const int* ids, const uint8_t* valid,
                                         int T, int E, int k, int eb, int ee, int t, int warp,
                                         int lane, unsigned int* status) {
  if (t < T && (valid == nullptr || valid[t])) {
    for (int j = 0; j < k; ++j) {
      const int e = ids[(size_t)t * k + j];
      if (e < 0 || e >= E) {
        if (status != nullptr) atomicOr(status, MOE_DEV_BAD_EXPERT_ID);
        continue;
      }
      if (e >= eb && e < ee) atomicOr(&bits[e][warp], 1u << lane);
    }
  }
}

__global__ void __launch_bounds__(1024, 1) route_kernel(const int* __restrict__ ids,
                                                        const uint8_t* __restrict__ valid, int T,
                                                        int E, int k, int S, int eb, int ee,
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
    set_bits(bits, ids, valid, T, E, k, eb, ee, t, warp, lane, status);
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

  // pass 2: ranks, permutation, inverse, row -> token (with one chunk, the bitmaps of
  // pass 1 are still in place)
  for (int c = 0; c < nchunks; ++c) {
    const int t = c * kChunk + tid;
    const bool ok = t < T && (valid == nullptr || valid[t]);
    const uint32_t vb = __ballot_sync(0xffffffffu, ok);
    if (nchunks > 1) {
      for (int i = tid; i < E * 32; i += blockDim.x) bits[i >> 5][i & 31] = 0u;
      __syncthreads();
      set_bits(bits, ids, valid, T, E, k, eb, ee, t, warp, lane, nullptr);
      if (lane == 0) wvalid[warp] = __popc(vb);
      __syncthreads();
    }
    if (t < T) {
      if (ok) {
        for (int j = 0; j < k; ++j) {
          const int e = ids[(size_t)t * k + j];
          if (e < eb || e >= ee || e >= E) {
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

// The same permutation for many chunks in parallel: (1) each chunk counts its
// pairs per expert and its valid tokens, (2) one block turns the counts into
// group offsets and per-chunk bases (expert-major, chunk-minor, so tokens stay
// ascending inside an expert), (3) each chunk ranks and scatters its pairs, four
// blocks to a chunk (each builds the chunk's bitmaps and stores the pairs of a
// quarter of its tokens).  Identical results to route_kernel.
__global__ void __launch_bounds__(1024, 1) route_count_kernel(const int* __restrict__ ids,
                                                              const uint8_t* __restrict__ valid,
                                                              int T, int E, int k, int eb, int ee,
                                                              int* __restrict__ chunk_cnt,
                                                              int* __restrict__ chunk_valid,
                                                              unsigned int* status) {
  __shared__ uint32_t bits[kMaxExperts][32];
  __shared__ int wvalid[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, c = blockIdx.x;
  for (int i = tid; i < E * 32; i += blockDim.x) bits[i >> 5][i & 31] = 0u;
  __syncthreads();
  const int t = c * kChunk + tid;
  set_bits(bits, ids, valid, T, E, k, eb, ee, t, warp, lane, status);
  const uint32_t vb = __ballot_sync(0xffffffffu, t < T && (valid == nullptr || valid[t]));
  if (lane == 0) wvalid[warp] = __popc(vb);
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    int s = 0;
    for (int w = 0; w < 32; ++w) s += __popc(bits[e][w]);
    chunk_cnt[(size_t)c * E + e] = s;
  }
  if (tid == 0) {
    int s = 0;
    for (int w = 0; w < 32; ++w) s += wvalid[w];
    chunk_valid[c] = s;
  }
}

__global__ void __launch_bounds__(1024, 1) route_scan_kernel(const int* __restrict__ chunk_cnt,
                                                             const int* __restrict__ chunk_valid,
                                                             int nchunks, int E, int S,
                                                             int* __restrict__ chunk_base,
                                                             int* __restrict__ vbase,
                                                             int* __restrict__ group_offsets) {
  __shared__ int tot[kMaxExperts];
  __shared__ int s_valid;
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) {
    int s = 0;
    for (int c = 0; c < nchunks; ++c) s += chunk_cnt[(size_t)c * E + e];
    tot[e] = s;
  }
  if (tid == 0) {
    int s = 0;
    for (int c = 0; c < nchunks; ++c) {
      vbase[c] = s;
      s += chunk_valid[c];
    }
    s_valid = s;
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int e = 0; e < E; ++e) {
      const int v = tot[e];
      tot[e] = acc;
      group_offsets[e] = acc;
      acc += v;
    }
    group_offsets[E] = acc;
    if (S) group_offsets[E + 1] = acc + s_valid;
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    int run = tot[e];
    for (int c = 0; c < nchunks; ++c) {
      chunk_base[(size_t)c * E + e] = run;
      run += chunk_cnt[(size_t)c * E + e];
    }
  }
}

__global__ void __launch_bounds__(1024, 1) route_scatter_kernel(
    const int* __restrict__ ids, const uint8_t* __restrict__ valid, int T, int E, int k, int S,
    int eb, int ee, const int* __restrict__ chunk_base, const int* __restrict__ vbase,
    const int* __restrict__ group_offsets, int* __restrict__ perm, int* __restrict__ inv,
    int* __restrict__ row_token, unsigned int* status) {
  __shared__ uint32_t bits[kMaxExperts][32];
  __shared__ int wvalid[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = blockIdx.x / kScatterSplit, part = blockIdx.x % kScatterSplit;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int i = tid; i < E * 32; i += blockDim.x) bits[i >> 5][i & 31] = 0u;
  __syncthreads();
  const int t = c * kChunk + tid;
  set_bits(bits, ids, valid, T, E, k, eb, ee, t, warp, lane, status);
  const bool ok = t < T && (valid == nullptr || valid[t]);
  const uint32_t vb = __ballot_sync(0xffffffffu, ok);
  if (lane == 0) wvalid[warp] = __popc(vb);
  __syncthreads();
  // every block of the chunk builds its bitmaps; each stores the pairs of its own
  // share of the chunk's tokens (the scattered stores are spread over more SMs)
  if (tid / (kChunk / kScatterSplit) != part || t >= T) return;
  const int ks = k + S;
  if (!ok) {
    for (int j = 0; j < ks; ++j) inv[(size_t)t * ks + j] = -1;
    return;
  }
  for (int j = 0; j < k; ++j) {
    const int e = ids[(size_t)t * k + j];
    if (e < eb || e >= ee || e >= E) {
      inv[(size_t)t * ks + j] = -1;
      continue;
    }
    int r = chunk_base[(size_t)c * E + e];
    for (int w = 0; w < warp; ++w) r += __popc(bits[e][w]);
    r += __popc(bits[e][warp] & lt_mask);
    perm[r] = t * k + j;
    inv[(size_t)t * ks + j] = r;
    row_token[r] = t;
  }
  if (S) {
    int vr = vbase[c] + __popc(vb & lt_mask);
    for (int w = 0; w < warp; ++w) vr += wvalid[w];
    const int pos = group_offsets[E] + vr;
    inv[(size_t)t * ks + k] = pos;
    row_token[pos] = t;
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

// Eight consecutive expert outputs as loaded: two 16-byte vectors of fp32 rows, or
// one of bf16 rows (FP8 path), widened to fp32 when summed.
template <typename YT> struct Vec8;
template <> struct Vec8<float> {
  float4 a, b;
};
template <> struct Vec8<__nv_bfloat16> {
  uint4 r;
};
__device__ __forceinline__ Vec8<float> ld8(const float* y8) {
  Vec8<float> v;
  v.a = reinterpret_cast<const float4*>(y8)[0];
  v.b = reinterpret_cast<const float4*>(y8)[1];
  return v;
}
__device__ __forceinline__ Vec8<__nv_bfloat16> ld8(const __nv_bfloat16* y8) {
  Vec8<__nv_bfloat16> v;
  v.r = *reinterpret_cast<const uint4*>(y8);
  return v;
}
__device__ __forceinline__ float elem8(const Vec8<float>& v, int i) {
  return i < 4 ? (i == 0 ? v.a.x : i == 1 ? v.a.y : i == 2 ? v.a.z : v.a.w)
               : (i == 4 ? v.b.x : i == 5 ? v.b.y : i == 6 ? v.b.z : v.b.w);
}
__device__ __forceinline__ float elem8(const Vec8<__nv_bfloat16>& v, int i) {
  const uint32_t w = i < 2 ? v.r.x : i < 4 ? v.r.y : i < 6 ? v.r.z : v.r.w;
  return __uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));   // bf16 -> fp32 is exact
}

// MAXKS bounds k + S at compile time, so that the variant for up to four rows a token
// (decode: top-3 with a shared expert) keeps only four row vectors in registers and
// runs at twice the occupancy of the general one.  With bf16 expert outputs (FP8
// weights) the registers are capped for three resident blocks an SM.
template <typename YT, bool F32OUT, int MAXKS>
__global__ void __launch_bounds__(256, sizeof(YT) == 2 ? 3 : 1)
    combine_kernel(const YT* __restrict__ y, int H, const int* __restrict__ inv,
                   const float* __restrict__ w, const uint8_t* __restrict__ valid, int T, int k,
                   int S, const CombineOut co) {
  __shared__ int rows[kMaxTopK + 1];
  __shared__ float wts[kMaxTopK];
  const int ks = k + S;
  const int nv = H / 8;
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    const bool ok = valid == nullptr || valid[t];
    if (threadIdx.x < ks) rows[threadIdx.x] = ok ? inv[(size_t)t * ks + threadIdx.x] : -1;
    if (threadIdx.x < k) wts[threadIdx.x] = ok ? w[(size_t)t * k + threadIdx.x] : 0.f;
    __syncthreads();
    uint4* dst16 = nullptr;
    float4* dst32 = nullptr;
    if (F32OUT) {
      const int owner = t / co.rows_per_rank, lt = t - owner * co.rows_per_rank;
      float* base = co.dst[0];
#pragma unroll
      for (int r = 1; r < kMaxTpRanks; ++r)
        if (owner == r) base = co.dst[r];
      dst32 = reinterpret_cast<float4*>(base + ((size_t)co.slot * co.rows_per_rank + lt) * H);
    } else {
      dst16 = reinterpret_cast<uint4*>(co.bf16 + (size_t)t * H);
    }
    for (int v = threadIdx.x; v < nv; v += blockDim.x) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (ok) {
        // every row's vector is requested before the sums (one round trip, not k+S),
        // and the sums keep their order: j ascending, then the shared expert
        // (named registers rather than an array, which the compiler put in local memory)
        static_assert(kMaxTopK == 8, "one register set per possible row below");
        const YT* yv = y + (size_t)v * 8;
#define MOE_LD(J) \
  Vec8<YT> r##J;  \
  if (J < MAXKS && J < ks && rows[J] >= 0) r##J = ld8(yv + (size_t)rows[J] * H);
        MOE_LD(0) MOE_LD(1) MOE_LD(2) MOE_LD(3) MOE_LD(4) MOE_LD(5) MOE_LD(6) MOE_LD(7) MOE_LD(8)
#undef MOE_LD
#define MOE_FMA(J)                                                                 \
  if (J < MAXKS && J < k && rows[J] >= 0) {                                        \
    _Pragma("unroll") for (int i = 0; i < 8; ++i) acc[i] =                         \
        fmaf(wts[J], elem8(r##J, i), acc[i]);                                      \
  }
        MOE_FMA(0) MOE_FMA(1) MOE_FMA(2) MOE_FMA(3) MOE_FMA(4) MOE_FMA(5) MOE_FMA(6) MOE_FMA(7)
#undef MOE_FMA
        // the shared expert's row (slot k), added last
#define MOE_SH(J)                                                                  \
  if (J < MAXKS && S && J == k && rows[J] >= 0) {                                  \
    _Pragma("unroll") for (int i = 0; i < 8; ++i) acc[i] += elem8(r##J, i);        \
  }
        MOE_SH(1) MOE_SH(2) MOE_SH(3) MOE_SH(4) MOE_SH(5) MOE_SH(6) MOE_SH(7) MOE_SH(8)
#undef MOE_SH
      }
      if (F32OUT) {
        dst32[2 * v] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        dst32[2 * v + 1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      } else {
        uint4 o;
        __nv_bfloat162* po = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i) po[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        dst16[v] = o;
      }
    }
    __syncthreads();
  }
}

template <typename YT, bool F32OUT, int MAXKS>
__global__ void __launch_bounds__(256)
    combine_flat_kernel(const YT* __restrict__ y, int H, const int* __restrict__ inv,
                   const float* __restrict__ w, const uint8_t* __restrict__ valid, int T, int k,
                   int S, const CombineOut co) {
  // one (token, 8-column vector) pair per thread and step: every thread of the grid
  // busy whatever the mix of valid and padding rows; a warp's 32 vectors mostly
  // share their token, so its index loads are broadcasts.  (With bf16 expert
  // outputs and nine rows a token, the per-token combine_kernel is faster.)
  const int ks = k + S;
  const int nv = H / 8;
  const long long total = (long long)T * nv;
  for (long long task = (long long)blockIdx.x * blockDim.x + threadIdx.x; task < total;
       task += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(task / nv);
    const int v = (int)(task - (long long)t * nv);
    const bool ok = valid == nullptr || valid[t];
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (ok) {
      const int* rows = inv + (size_t)t * ks;
      const float* wts = w + (size_t)t * k;
      // every row's vector is requested before the sums (one round trip, not k+S),
      // and the sums keep their order: j ascending, then the shared expert
      // (named registers rather than an array, which the compiler put in local memory)
      static_assert(kMaxTopK == 8, "one register set per possible row below");
      const YT* yv = y + (size_t)v * 8;
#define MOE_LD(J)                                              \
  Vec8<YT> r##J;                                               \
  const int row##J = (J < MAXKS && J < ks) ? rows[J] : -1;     \
  if (row##J >= 0) r##J = ld8(yv + (size_t)row##J * H);
      MOE_LD(0) MOE_LD(1) MOE_LD(2) MOE_LD(3) MOE_LD(4) MOE_LD(5) MOE_LD(6) MOE_LD(7) MOE_LD(8)
#undef MOE_LD
#define MOE_FMA(J)                                                                 \
  if (J < MAXKS && J < k && row##J >= 0) {                                         \
    const float wj = wts[J];                                                       \
    _Pragma("unroll") for (int i = 0; i < 8; ++i) acc[i] =                         \
        fmaf(wj, elem8(r##J, i), acc[i]);                                          \
  }
      MOE_FMA(0) MOE_FMA(1) MOE_FMA(2) MOE_FMA(3) MOE_FMA(4) MOE_FMA(5) MOE_FMA(6) MOE_FMA(7)
#undef MOE_FMA
      // the shared expert's row (slot k), added last
#define MOE_SH(J)                                                                  \
  if (J < MAXKS && S && J == k && row##J >= 0) {                                   \
    _Pragma("unroll") for (int i = 0; i < 8; ++i) acc[i] += elem8(r##J, i);        \
  }
      MOE_SH(1) MOE_SH(2) MOE_SH(3) MOE_SH(4) MOE_SH(5) MOE_SH(6) MOE_SH(7) MOE_SH(8)
#undef MOE_SH
    }
    if (F32OUT) {
      const int owner = t / co.rows_per_rank, lt = t - owner * co.rows_per_rank;
      float* base = co.dst[0];
#pragma unroll
      for (int r = 1; r < kMaxTpRanks; ++r)
        if (owner == r) base = co.dst[r];
      float4* dst32 =
          reinterpret_cast<float4*>(base + ((size_t)co.slot * co.rows_per_rank + lt) * H);
      dst32[2 * v] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      dst32[2 * v + 1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    } else {
      uint4 o;
      __nv_bfloat162* po = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
      for (int i = 0; i < 4; ++i) po[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
      reinterpret_cast<uint4*>(co.bf16 + (size_t)t * H)[v] = o;
    }
  }
}

// Owner side of the tensor-parallel reduction: the slab holds one fp32 partial
// row per rank for each of this rank's rows; they are summed in rank order (the
// same order on every owner) and rounded once to bf16.
__global__ void __launch_bounds__(256) reduce_slots_kernel(const float* __restrict__ slots,
                                                           int n_slots, int rows, int H,
                                                           const uint8_t* __restrict__ valid,
                                                           __nv_bfloat16* __restrict__ out) {
  const int nv = H / 8;
  const size_t slab = (size_t)rows * H;
  for (int t = blockIdx.x; t < rows; t += gridDim.x) {
    const bool ok = valid == nullptr || valid[t];
    uint4* dst = reinterpret_cast<uint4*>(out + (size_t)t * H);
    for (int v = threadIdx.x; v < nv; v += blockDim.x) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (ok) {
        for (int g = 0; g < n_slots; ++g) {
          const float4* src =
              reinterpret_cast<const float4*>(slots + g * slab + (size_t)t * H) + 2 * v;
          const float4 a = src[0], b = src[1];
          acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
          acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
        }
      }
      uint4 o;
      __nv_bfloat162* po = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
      for (int i = 0; i < 4; ++i) po[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
      dst[v] = o;
    }
  }
}

// Owner side of the per-pair return: slot j < k of row t holds the unweighted output
// row of t's j-th routed expert (sent by the rank that owns that expert), slots
// k .. k + n_extra - 1 the shared expert's shares; the sum takes the same order as
// the one-GPU combine (fused multiply-adds over j ascending, then the shared rows),
// so on one rank it equals the plain forward bit for bit.
__global__ void __launch_bounds__(256) reduce_pairs_kernel(const float* __restrict__ slab, int k,
                                                           int n_extra, int rows, int H,
                                                           const float* __restrict__ w,
                                                           const uint8_t* __restrict__ valid,
                                                           __nv_bfloat16* __restrict__ out) {
  const int nv = H / 8;
  const size_t per_slot = (size_t)rows * H;
  for (int t = blockIdx.x; t < rows; t += gridDim.x) {
    const bool ok = valid == nullptr || valid[t];
    uint4* dst = reinterpret_cast<uint4*>(out + (size_t)t * H);
    for (int v = threadIdx.x; v < nv; v += blockDim.x) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (ok) {
        for (int j = 0; j < k + n_extra; ++j) {
          const float4* src =
              reinterpret_cast<const float4*>(slab + j * per_slot + (size_t)t * H) + 2 * v;
          const float4 a = src[0], b = src[1];
          const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
          if (j < k) {
            const float wj = w[(size_t)t * k + j];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = fmaf(wj, f[i], acc[i]);
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] += f[i];
          }
        }
      }
      uint4 o;
      __nv_bfloat162* po = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
      for (int i = 0; i < 4; ++i) po[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
      dst[v] = o;
    }
  }
}

// FP8 path, activation quantisation: a warp takes up to four 1x128 groups of one
// valid token (eight lanes a group, 16 consecutive values a lane, loads issued
// together), computes for each s = amax / 448 (1 if amax = 0) and the e4m3 codes of
// x / s (fp32 division, round to nearest even, saturating), once per token, and
// stores codes and scale straight into every permuted row the token occupies (its k
// routed rows and the shared one, from the inverse permutation), one 512-byte store
// of the warp per row: the GEMM's activation rows are written once, with no
// per-token copy to gather from.
constexpr int kQuantGroupsPerWarp = 4;

__global__ void __launch_bounds__(256) quant_scatter_kernel(const __nv_bfloat16* __restrict__ x,
                                                            const uint8_t* __restrict__ valid,
                                                            int T, int H,
                                                            const int* __restrict__ inv, int ks,
                                                            uint8_t* __restrict__ xp,
                                                            float* __restrict__ sxp) {
  const int lane = threadIdx.x & 31;
  const int groups = H / 128;
  const int chunks = (groups + kQuantGroupsPerWarp - 1) / kQuantGroupsPerWarp;
  const long long nwarps = (long long)gridDim.x * (blockDim.x / 32);
  for (long long wc = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
       wc < (long long)T * chunks; wc += nwarps) {
    const int t = (int)(wc / chunks);
    const int g0 = (int)(wc - (long long)t * chunks) * kQuantGroupsPerWarp;
    if (valid != nullptr && !valid[t]) continue;
    const int ng = min(kQuantGroupsPerWarp, groups - g0);
    // lane l takes 16 consecutive values of group u = l / 8 (eight lanes a group), so
    // that a row's four groups leave the warp as one 512-byte store per row
    const int u = lane >> 3;
    const bool act = u < ng;
    const size_t col = (size_t)g0 * 128 + (size_t)lane * 16;
    uint4 raw[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
    if (act) {
      const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H + col);
      raw[0] = src[0];
      raw[1] = src[1];
    }
    int rows[kMaxTopK + 1];
#pragma unroll
    for (int j = 0; j < kMaxTopK + 1; ++j) rows[j] = j < ks ? inv[(size_t)t * ks + j] : -1;
    float v[16];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t w4[4] = {raw[h].x, raw[h].y, raw[h].z, raw[h].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 pr = *reinterpret_cast<const __nv_bfloat162*>(&w4[i]);
        v[8 * h + 2 * i] = __low2float(pr);
        v[8 * h + 2 * i + 1] = __high2float(pr);
      }
    }
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(v[i]));
#pragma unroll
    for (int off = 4; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
    if (!act) continue;
    const float sc = a > 0.f ? __fdiv_rn(a, 448.f) : 1.f;
    uint32_t packed[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      packed[w] = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        packed[w] |= (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(v[4 * w + i], sc), __NV_SATFINITE,
                                                     __NV_E4M3)
                     << (8 * i);
    }
    const uint4 q = make_uint4(packed[0], packed[1], packed[2], packed[3]);
#pragma unroll
    for (int j = 0; j < kMaxTopK + 1; ++j) {
      const int r = rows[j];
      if (r < 0) continue;
      *reinterpret_cast<uint4*>(xp + (size_t)r * H + col) = q;
      if ((lane & 7) == 0) sxp[(size_t)r * groups + g0 + u] = sc;
    }
  }
}

}  // namespace

int route_scratch_ints(int max_tokens, int E) {
  const int nchunks = (max_tokens + kChunk - 1) / kChunk;
  return nchunks * (2 * E + 2);
}

cudaError_t launch_route(const int* ids, const uint8_t* valid, int T, int E, int k, int S,
                         int eb, int ee, int* group_offsets, int* perm, int* inv, int* row_token,
                         unsigned int* status, int* scratch, cudaStream_t st) {
  const int nchunks = (T + kChunk - 1) / kChunk;
  if (nchunks <= 1 || scratch == nullptr) {
    route_kernel<<<1, 1024, 0, st>>>(ids, valid, T, E, k, S, eb, ee, group_offsets, perm, inv,
                                     row_token, status);
    return cudaGetLastError();
  }
  int* chunk_cnt = scratch;                        // [nchunks][E]
  int* chunk_base = chunk_cnt + (size_t)nchunks * E;   // [nchunks][E]
  int* chunk_valid = chunk_base + (size_t)nchunks * E; // [nchunks]
  int* vbase = chunk_valid + nchunks;                  // [nchunks]
  route_count_kernel<<<nchunks, 1024, 0, st>>>(ids, valid, T, E, k, eb, ee, chunk_cnt,
                                               chunk_valid, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  route_scan_kernel<<<1, 1024, 0, st>>>(chunk_cnt, chunk_valid, nchunks, E, S, chunk_base, vbase,
                                        group_offsets);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // set_bits reports a bad expert id once in the count pass; the scatter pass skips it quietly
  route_scatter_kernel<<<nchunks * kScatterSplit, 1024, 0, st>>>(
      ids, valid, T, E, k, S, eb, ee, chunk_base, vbase, group_offsets, perm, inv, row_token,
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

// up to four rows a token (k + S <= 4) with the small-register variant
template <typename YT, bool F32OUT>
void launch_combine_rows(const YT* y, int H, const int* inv, const float* w,
                         const uint8_t* valid, int T, int k, int S, const CombineOut& out,
                         int grid, cudaStream_t st) {
  if (k + S <= 4)
    combine_kernel<YT, F32OUT, 4><<<grid, 256, 0, st>>>(y, H, inv, w, valid, T, k, S, out);
  else
    combine_kernel<YT, F32OUT, kMaxTopK + 1><<<grid, 256, 0, st>>>(y, H, inv, w, valid, T, k,
                                                                  S, out);
}

template <bool F32OUT>
void launch_combine_flat(const float* y, int H, const int* inv, const float* w,
                         const uint8_t* valid, int T, int k, int S, const CombineOut& out,
                         cudaStream_t st) {
  const long long blocks = ((long long)T * (H / 8) + 255) / 256;
  const int grid = (int)(blocks < 1 ? 1 : blocks > 148 * 16 ? 148 * 16 : blocks);
  if (k + S <= 4)
    combine_flat_kernel<float, F32OUT, 4><<<grid, 256, 0, st>>>(y, H, inv, w, valid, T, k, S,
                                                                out);
  else
    combine_flat_kernel<float, F32OUT, kMaxTopK + 1><<<grid, 256, 0, st>>>(y, H, inv, w, valid,
                                                                          T, k, S, out);
}

// fp32 expert outputs (bf16 weights): one (token, vector) pair a thread, which keeps a
// batch that is mostly padding rows (the DP-padded gather) as busy as a full one
cudaError_t launch_combine(const float* y, int H, const int* inv, const float* w,
                           const uint8_t* valid, int T, int k, int S, const CombineOut& out,
                           cudaStream_t st) {
  if (out.bf16 != nullptr)
    launch_combine_flat<false>(y, H, inv, w, valid, T, k, S, out, st);
  else
    launch_combine_flat<true>(y, H, inv, w, valid, T, k, S, out, st);
  return cudaGetLastError();
}

cudaError_t launch_combine_bf16y(const __nv_bfloat16* y, int H, const int* inv, const float* w,
                                 const uint8_t* valid, int T, int k, int S, const CombineOut& out,
                                 cudaStream_t st) {
  int grid = T < 148 * 16 ? T : 148 * 16;
  if (grid < 1) grid = 1;
  if (out.bf16 != nullptr)
    launch_combine_rows<__nv_bfloat16, false>(y, H, inv, w, valid, T, k, S, out, grid, st);
  else
    launch_combine_rows<__nv_bfloat16, true>(y, H, inv, w, valid, T, k, S, out, grid, st);
  return cudaGetLastError();
}

cudaError_t launch_reduce_slots(const float* slots, int n_slots, int rows, int H,
                                const uint8_t* valid, __nv_bfloat16* out, cudaStream_t st) {
  int grid = rows < 148 * 16 ? rows : 148 * 16;
  if (grid < 1) grid = 1;
  reduce_slots_kernel<<<grid, 256, 0, st>>>(slots, n_slots, rows, H, valid, out);
  return cudaGetLastError();
}

cudaError_t launch_reduce_pairs(const float* slab, int k, int n_extra, int rows, int H,
                                const float* w, const uint8_t* valid, __nv_bfloat16* out,
                                cudaStream_t st) {
  const int grid = rows < 4096 ? rows : 4096;
  reduce_pairs_kernel<<<grid, 256, 0, st>>>(slab, k, n_extra, rows, H, w, valid, out);
  return cudaGetLastError();
}

cudaError_t launch_quant_scatter(const __nv_bfloat16* x, const uint8_t* valid, int T, int H,
                                 const int* inv, int ks, uint8_t* xp, float* sxp, int num_sms,
                                 cudaStream_t st) {
  const int chunks = (H / 128 + kQuantGroupsPerWarp - 1) / kQuantGroupsPerWarp;
  const long long warps = (long long)T * chunks;
  long long g1 = (warps + 7) / 8;
  if (g1 > (long long)num_sms * 16) g1 = (long long)num_sms * 16;
  if (g1 < 1) g1 = 1;
  quant_scatter_kernel<<<(int)g1, 256, 0, st>>>(x, valid, T, H, inv, ks, xp, sxp);
  return cudaGetLastError();
}

}  // namespace moe
