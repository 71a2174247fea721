// Router logits on the tensor cores: l[t,e] = sum_h x[t,h] Wr[e,h] with fp32
// router weights and bf16 hidden states (Step3 推論最適化 (MI308X vs H20), §背景:
// each token scores all experts and keeps 3 of 48).
//
// The tensor core multiplies bf16 (or lower) operands, so the fp32 weights are
// split exactly into three bf16 parts, Wr = W1 + W2 + W3 (each part the bf16
// rounding of what the previous ones left; 3 x 8 significand bits cover
// fp32's 24), and the three products x W1, x W2, x W3 accumulate into one fp32
// accumulator: every product of a bf16 x and a bf16 part is exact in fp32, so
// the result is the fp32-accumulated dot product with the full fp32 weights.
//
// router_tc_kernel: one CTA per (128-token tile, up-to-128-expert tile, K
// split); tokens on the MMA's M side, experts on N; TMA ring of 64-wide K
// blocks (x tile + the three weight parts), accumulator in TMEM, written as
// fp32 partial sums per split, which the top-k kernel adds in split order.
// Token tiles without a valid row are skipped.
#include <cudaTypedefs.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int RBM = 128;           // tokens per tile
constexpr int RBN = 128;           // experts per tile
constexpr int RBK = 64;            // bf16 K elements per stage (128 bytes)
constexpr int RSTAGES = 3;
constexpr int RA_BYTES = RBM * RBK * 2;          // 16 KB
constexpr int RB_BYTES = 3 * RBN * RBK * 2;      // 48 KB (three weight parts)
constexpr int RSMEM = RSTAGES * (RA_BYTES + RB_BYTES) + 1024 + 1024;
constexpr int RThreads = 192;
constexpr unsigned long long kRouterWaitNs = 2000000000ull;

__global__ void __launch_bounds__(256) split_router_weights_kernel(const float* __restrict__ Wr,
                                                                   int E, int E_pad, int H,
                                                                   __nv_bfloat16* __restrict__ W3) {
  const size_t n = (size_t)E_pad * H;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const int e = (int)(i / H);
    const float w = e < E ? Wr[i] : 0.f;
    const __nv_bfloat16 b1 = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(b1);          // exact
    const __nv_bfloat16 b2 = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(b2);          // exact
    const __nv_bfloat16 b3 = __float2bfloat16_rn(r2);
    W3[i] = b1;
    W3[n + i] = b2;
    W3[2 * n + i] = b3;
  }
}

struct RParams {
  int T, E, E_pad, kb_total, kb_per_split;
  const uint8_t* valid;
  float* partial;                  // [splits, T, E]
  unsigned int* status;
  unsigned int timeout_bit;
};

__global__ void __launch_bounds__(RThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const RParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* a_smem = base;
  uint8_t* b_smem = base + RSTAGES * RA_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + RSTAGES * (RA_BYTES + RB_BYTES));
  uint64_t* full = bars;
  uint64_t* empty = bars + RSTAGES;
  uint64_t* tfull = bars + 2 * RSTAGES;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tfull + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * RBM, e0 = blockIdx.y * RBN, split = blockIdx.z;
  const int n = min(RBN, p.E_pad - e0);              // multiple of 16
  const int kb0 = split * p.kb_per_split;
  const int kb1 = min(p.kb_total, kb0 + p.kb_per_split);

  // skip token tiles that hold no valid row (all CTAs of a tile agree)
  int mine = 0;
  for (int r = threadIdx.x; r < RBM; r += blockDim.x) {
    const int t = t0 + r;
    if (t < p.T && (p.valid == nullptr || p.valid[t])) mine = 1;
  }
  if (!__syncthreads_or(mine) || kb0 >= kb1) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < RSTAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(tfull), 1);
    fence_mbarrier_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), RBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();     // x and the weight parts are re-read by other CTAs
      int stage = 0;
      uint32_t phase = 0, issued = 0, parity = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait_sleep(smem_u32(&empty[stage]), phase ^ 1u, kRouterWaitNs, p.status,
                             p.timeout_bit))
          break;
        const uint32_t fb = smem_u32(&full[stage]);
        mbar_arrive_expect_tx(fb, RA_BYTES + RB_BYTES);
        tma_load_2d(smem_u32(a_smem + stage * RA_BYTES), &tmX, kb * RBK, t0, fb, pol);
        const uint32_t b_dst = smem_u32(b_smem + stage * RB_BYTES);
#pragma unroll
        for (int s = 0; s < 3; ++s)
          tma_load_2d(b_dst + s * RBN * RBK * 2, &tmW, kb * RBK, s * p.E_pad + e0, fb, pol);
        issued |= 1u << stage;
        parity = (parity & ~(1u << stage)) | (phase << stage);
        if (++stage == RSTAGES) { stage = 0; phase ^= 1u; }
      }
      for (int s = 0; s < RSTAGES; ++s)
        if ((issued >> s) & 1u)
          mbar_wait_sleep(smem_u32(&full[s]), (parity >> s) & 1u, kRouterWaitNs, p.status,
                          p.timeout_bit);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_m128(n);
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait_sleep(smem_u32(&full[stage]), phase, kRouterWaitNs, p.status,
                             p.timeout_bit))
          break;   // status bit set; commit below still drains what was issued
        tc_fence_after();
        const uint64_t a_desc = smem_desc_sw128(smem_u32(a_smem + stage * RA_BYTES));
#pragma unroll
        for (int kk = 0; kk < RBK / 16; ++kk) {
#pragma unroll
          for (int s = 0; s < 3; ++s) {
            const uint64_t b_desc =
                smem_desc_sw128(smem_u32(b_smem + stage * RB_BYTES + s * RBN * RBK * 2));
            umma_bf16(tmem_base, a_desc + 2 * kk, b_desc + 2 * kk, idesc,
                      (kb > kb0 || kk > 0 || s > 0) ? 1u : 0u);
          }
        }
        umma_commit(smem_u32(&empty[stage]));
        if (++stage == RSTAGES) { stage = 0; phase ^= 1u; }
      }
      // tfull also marks that every MMA has finished: wait for it before the
      // tensor memory is released
      umma_commit(smem_u32(tfull));
      mbar_wait_sleep(smem_u32(tfull), 0, kRouterWaitNs, p.status, p.timeout_bit);
    }
    __syncwarp();
  } else {
    // epilogue: warp w reads TMEM lanes 32*(w%4).. = tokens t0 + 32*(w%4) + lane
    const int q = warp & 3;
    const bool done = mbar_wait_sleep_warp(smem_u32(tfull), 0, kRouterWaitNs, p.status,
                                           p.timeout_bit);
    tc_fence_after();
    const int t = t0 + q * 32 + lane;
    float* out = p.partial + ((size_t)split * p.T + t) * p.E + e0;
    if (done) {
      for (int c0 = 0; c0 < n; c0 += 16) {
        float v[16];
        tmem_ld_16(tmem_base + ((uint32_t)(q * 32) << 16) + c0, v);
        if (t < p.T) {
          // 16-byte stores where four experts of the row exist (the row is E floats,
          // 16-byte aligned when E is a multiple of 4), single floats otherwise
#pragma unroll
          for (int c = 0; c < 16; c += 4) {
            if ((p.E & 3) == 0 && e0 + c0 + c + 3 < p.E) {
              *reinterpret_cast<float4*>(out + c0 + c) =
                  make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
            } else {
#pragma unroll
              for (int i = 0; i < 4; ++i)
                if (e0 + c0 + c + i < p.E) out[c0 + c + i] = v[c + i];
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, RBN);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encoder_r() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool map_bf16_rows(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer) {
  auto enc = encoder_r();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {(cuuint32_t)RBK, 128};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int router_padded_experts(int E) { return (E + 15) / 16 * 16; }

void router_split_plan(int T, int E, int H, int num_sms, int partial_rows, int* splits_out,
                       int* kb_per_split_out) {
  const int kb_total = H / RBK;
  const int tiles = ((T + RBM - 1) / RBM) * ((router_padded_experts(E) + RBN - 1) / RBN);
  int splits = (2 * num_sms + tiles - 1) / tiles;
  if (splits < 1) splits = 1;
  // as many splits as the partial-sum buffer holds rows of this batch
  const int cap = T > 0 ? partial_rows / T : kRouterSplitMax;
  if (splits > cap) splits = cap;
  if (splits > kb_total) splits = kb_total;
  const int per = (kb_total + splits - 1) / splits;
  *kb_per_split_out = per;
  *splits_out = (kb_total + per - 1) / per;        // every split gets at least one K block
}

cudaError_t prepare_router_kernel() {
  return cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              RSMEM);
}

cudaError_t launch_split_router_weights(const float* Wr, int E, int H, __nv_bfloat16* W3,
                                        int num_sms, cudaStream_t st) {
  split_router_weights_kernel<<<num_sms * 4, 256, 0, st>>>(Wr, E, router_padded_experts(E), H,
                                                           W3);
  return cudaGetLastError();
}

cudaError_t launch_router_logits_tc(const __nv_bfloat16* x, const uint8_t* valid, int T, int H,
                                    const __nv_bfloat16* W3, int E, float* partial, int splits,
                                    int kb_per_split, unsigned int* status, cudaStream_t st) {
  const int E_pad = router_padded_experts(E);
  CUtensorMap tmX, tmW;
  if (!map_bf16_rows(&tmX, x, H, T) || !map_bf16_rows(&tmW, W3, H, (uint64_t)3 * E_pad))
    return cudaErrorInvalidValue;
  RParams p;
  p.T = T;
  p.E = E;
  p.E_pad = E_pad;
  p.kb_total = H / RBK;
  p.kb_per_split = kb_per_split;
  p.valid = valid;
  p.partial = partial;
  p.status = status;
  p.timeout_bit = MOE_DEV_WAIT_TIMEOUT_ROUTER;
  dim3 g((T + RBM - 1) / RBM, (E_pad + RBN - 1) / RBN, splits);
  router_tc_kernel<<<g, RThreads, RSMEM, st>>>(tmX, tmW, p);
  return cudaGetLastError();
}

}  // namespace moe
