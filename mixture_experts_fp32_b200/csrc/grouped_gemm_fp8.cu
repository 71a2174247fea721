// Grouped expert GEMMs with e4m3 operands and fp32 block scales on tcgen05.
//
// The mixed BF16 / FP8 block-scale arithmetic of the pages (Step3 推論最適化
// (MI308X vs H20), §最適化技術; "GEMM à l'échelle bloc", AMD Instinct MI355X :
// ATOM, kernels fusionnés et montée en charge, introduction): weights carry one
// fp32 scale per 128x128 block, activations one per 1x128 group, so
//
//   acc[m, n] = sum_kb  s_w[m/128, kb] * s_a[n, kb] * sum_{k in kb} qw[m, k] * qa[n, k].
//
// The scale changes every 128 K, and arbitrary fp32 scales cannot be given to
// the tensor core's block-scaled kinds (they take power-of-two scales), so each
// 128-wide K block is multiplied (kind::f8f6f4, exact products, fp32 sums) into
// a fresh tensor-memory partial, and the epilogue warps fold every partial into
// fp32 register accumulators with its scale product ("promotion").  Two partial
// buffers let the tensor core run one K block ahead of the promotion.
//
//   gated: a tile owns 128 gate rows and the matching 128 up rows of one expert
//          (one 128-row scale block each) and up to 128 rows of activations;
//          after the last K block h = silu(g) * u is quantised per 1x128 group
//          (the tile's 128 columns of h are exactly one group) into e4m3 codes
//          with an fp32 scale, ready for the down GEMM.
//   down:  a tile owns 128 output features (one scale block) and up to 256
//          rows; y is written in bf16.
//
// Warp roles (576 threads): warp 0 issues TMA loads, warp 1 owns tensor memory
// and issues the MMAs, warps 2-17 promote and finish (warp w reads TMEM lanes
// 32*(w%4)... and one quarter of the tile's columns).  Waits are bounded.
#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int BK = 128;           // e4m3 elements (= bytes) per K block: one scale group
constexpr int kEpiWarps = 16;
constexpr int kThreads = 64 + kEpiWarps * 32;
constexpr uint32_t kTmemCols = 512;
constexpr int kPartStride = 256;  // TMEM columns between the two partial buffers
constexpr unsigned long long kTeardownLimitNs = 1000000000ull;

template <bool GATED>
struct Cfg8 {
  static constexpr int BN = 128;                          // activation rows per tile
  static constexpr int COLS = BN / 4;                     // columns per epilogue warp
  static constexpr int A_BYTES = (GATED ? 2 : 1) * BM * BK;
  static constexpr int B_BYTES = BN * BK;
  static constexpr int STAGES = 4;
  static constexpr int DATA_BYTES = STAGES * (A_BYTES + B_BYTES);
  static constexpr int RED_BYTES = GATED ? 2 * 4 * BN * 4 : 0;   // column maxima [2][4][BN]
  static constexpr int SMEM_BYTES = DATA_BYTES + RED_BYTES + 1024 + 2048;
};

struct KParams8 {
  const int* group_offsets;
  int E, G;
  int kb_routed, kb_shared;
  int rows_per_expert;
  int m_routed, m_shared;
  int up_routed, up_shared;
  const float* sa_routed;
  const float* sa_shared;
  const float* sb;
  void* d;
  float* sd;
  int ldd;
  int R_cap;
  unsigned int* status;
  unsigned int timeout_bit;
  unsigned long long wait_limit_ns;
};

struct Tile8 {
  int g, m, row0, nrows, n_mma, k_blocks;
};

template <int BN>
__device__ __forceinline__ Tile8 decode_tile8(int t, const int* ts, const int* go,
                                              const KParams8& p) {
  int lo = 0, hi = p.G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (ts[mid] <= t) lo = mid; else hi = mid;
  }
  Tile8 ti;
  ti.g = lo;
  const int gbeg = go[lo], gend = go[lo + 1];
  const int nt = (gend - gbeg + BN - 1) / BN;
  const int local = t - ts[lo];
  ti.m = local / nt;
  const int n = local - ti.m * nt;
  ti.row0 = gbeg + n * BN;
  ti.nrows = min(BN, gend - ti.row0);
  ti.n_mma = (ti.nrows + 15) & ~15;
  ti.k_blocks = lo < p.E ? p.kb_routed : p.kb_shared;
  return ti;
}

__device__ __forceinline__ uint8_t e4m3_of(float v) {
  return (uint8_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

template <bool GATED>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_fp8_kernel(const __grid_constant__ CUtensorMap tmA,
                            const __grid_constant__ CUtensorMap tmAs,
                            const __grid_constant__ CUtensorMap tmB, const KParams8 p) {
  using C = Cfg8<GATED>;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* a_smem = base;
  uint8_t* b_smem = base + C::STAGES * C::A_BYTES;
  float* red = reinterpret_cast<float*>(base + C::DATA_BYTES);   // [tile parity][quadrant][column]
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + C::DATA_BYTES + C::RED_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* pfull = bars + 2 * C::STAGES;
  uint64_t* pempty = pfull + 2;
  uint64_t* teardown = pempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(teardown + 1);
  int* ts = reinterpret_cast<int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int* go = p.group_offsets;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&pfull[b]), 1);
      mbar_init(smem_u32(&pempty[b]), kEpiWarps);
    }
    mbar_init(smem_u32(teardown), 1);
    fence_mbarrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmAs);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 2) {
    int running = 0;
    for (int b0 = 0; b0 < p.G; b0 += 32) {
      const int g = b0 + lane;
      int cnt = 0;
      if (g < p.G) {
        const int rows = go[g + 1] - go[g];
        cnt = (g < p.E ? p.m_routed : p.m_shared) * ((rows + BN - 1) / BN);
      }
      int incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      if (g < p.G) ts[g] = running + incl - cnt;
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) ts[p.G] = running;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total = ts[p.G];

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_a = policy_evict_first();
      const uint64_t pol_b = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0, issued = 0, parity = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const Tile8 ti = decode_tile8<BN>(t, ts, go, p);
        const bool routed = ti.g < p.E;
        const CUtensorMap* am = routed ? &tmA : &tmAs;
        const int arow = (routed ? ti.g * p.rows_per_expert : 0) + ti.m * BM;
        const int up = routed ? p.up_routed : p.up_shared;
        const uint32_t bytes = C::A_BYTES + ti.n_mma * BK;
        for (int kb = 0; kb < ti.k_blocks; ++kb) {
          if (!mbar_wait_bounded(smem_u32(&empty[stage]), phase ^ 1u, p.wait_limit_ns, p.status,
                                 p.timeout_bit)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_arrive_expect_tx(fb, bytes);
          const uint32_t a_dst = smem_u32(a_smem + stage * C::A_BYTES);
          tma_load_2d(a_dst, am, kb * BK, arow, fb, pol_a);
          if (GATED) tma_load_2d(a_dst + BM * BK, am, kb * BK, arow + up, fb, pol_a);
          const uint32_t b_dst = smem_u32(b_smem + stage * C::B_BYTES);
          for (int nb = 0; nb < ti.n_mma / 16; ++nb)
            tma_load_2d(b_dst + nb * 16 * BK, &tmB, kb * BK, ti.row0 + nb * 16, fb, pol_b);
          issued |= 1u << stage;
          parity = (parity & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      for (int s = 0; s < C::STAGES; ++s)
        if ((issued >> s) & 1u)
          mbar_wait_bounded(smem_u32(&full[s]), (parity >> s) & 1u, kTeardownLimitNs, p.status,
                            p.timeout_bit);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t kcount = 0;          // K blocks issued so far: partial buffer = kcount & 1
      bool ok = true, any = false;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const Tile8 ti = decode_tile8<BN>(t, ts, go, p);
        const uint32_t idesc = idesc_e4m3_m128(ti.n_mma);
        for (int kb = 0; kb < ti.k_blocks; ++kb, ++kcount) {
          const uint32_t pb = kcount & 1u;
          const uint32_t use = kcount >> 1;
          if (!mbar_wait_bounded(smem_u32(&pempty[pb]), (use & 1u) ^ 1u, p.wait_limit_ns,
                                 p.status, p.timeout_bit) ||
              !mbar_wait_bounded(smem_u32(&full[stage]), phase, p.wait_limit_ns, p.status,
                                 p.timeout_bit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d0 = tmem_base + pb * kPartStride;
          const uint64_t a_desc = smem_desc_sw128(smem_u32(a_smem + stage * C::A_BYTES));
          const uint64_t au_desc = smem_desc_sw128(smem_u32(a_smem + stage * C::A_BYTES + BM * BK));
          const uint64_t b_desc = smem_desc_sw128(smem_u32(b_smem + stage * C::B_BYTES));
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            // +32 bytes per 32-element K step, in 16-byte units of the address field
            umma_e4m3(d0, a_desc + 2 * kk, b_desc + 2 * kk, idesc, kk != 0);
            if (GATED) umma_e4m3(d0 + BN, au_desc + 2 * kk, b_desc + 2 * kk, idesc, kk != 0);
          }
          umma_commit(smem_u32(&empty[stage]));
          umma_commit(smem_u32(&pfull[pb]));
          any = true;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (any) {
        umma_commit(smem_u32(teardown));
        mbar_wait_bounded(smem_u32(teardown), 0, kTeardownLimitNs, p.status, p.timeout_bit);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------- promotion and epilogue
    // Every epilogue warp walks the same tiles and, for gated tiles, passes one
    // named barrier per tile whatever happens; after an expired wait it keeps
    // walking with no further waits, loads or stores, so no barrier is missed.
    const int ew = warp - 2;
    const int q = warp & 3;               // TMEM lane quadrant
    const int cq = ew >> 2;               // column quarter of the tile
    const int c0 = cq * C::COLS;          // first tile column of this warp
    uint32_t kcount = 0;
    int tiles_done = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++tiles_done) {
      const Tile8 ti = decode_tile8<BN>(t, ts, go, p);
      const bool routed = ti.g < p.E;
      const int ncols = max(0, min(C::COLS, ti.n_mma - c0));   // multiple of 16
      const float* sw = routed ? p.sa_routed + (size_t)ti.g * (p.rows_per_expert / BM) *
                                                   ti.k_blocks
                               : p.sa_shared;
      const int rb_gate = ti.m;
      const int rb_up = ((routed ? p.up_routed : p.up_shared) / BM) + ti.m;
      float acc_g[C::COLS];
      float acc_u[GATED ? C::COLS : 1];
#pragma unroll
      for (int c = 0; c < C::COLS; ++c) acc_g[c] = 0.f;
#pragma unroll
      for (int c = 0; c < (GATED ? C::COLS : 1); ++c) acc_u[c] = 0.f;
      for (int kb = 0; kb < ti.k_blocks && ok; ++kb, ++kcount) {
        const uint32_t pb = kcount & 1u;
        const uint32_t use = kcount >> 1;
        if (!mbar_wait_bounded_warp(smem_u32(&pfull[pb]), use & 1u, p.wait_limit_ns, p.status,
                                    p.timeout_bit)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float swg = sw[(size_t)rb_gate * ti.k_blocks + kb];
        const float swu = GATED ? sw[(size_t)rb_up * ti.k_blocks + kb] : 0.f;
        const float* sb = p.sb + (size_t)kb * p.R_cap + ti.row0 + c0;
        const uint32_t tl = tmem_base + ((uint32_t)(q * 32) << 16) + pb * kPartStride + c0;
#pragma unroll
        for (int cc = 0; cc < C::COLS; cc += 8) {
          if (cc < ncols) {
            float sa[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) sa[c] = (c0 + cc + c < ti.nrows) ? sb[cc + c] : 0.f;
            float v[8];
            tmem_ld_8(tl + cc, v);
#pragma unroll
            for (int c = 0; c < 8; ++c) acc_g[cc + c] = fmaf(v[c], swg * sa[c], acc_g[cc + c]);
            if (GATED) {
              tmem_ld_8(tl + BN + cc, v);
#pragma unroll
              for (int c = 0; c < 8; ++c) acc_u[cc + c] = fmaf(v[c], swu * sa[c], acc_u[cc + c]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&pempty[pb]));
      }

      const int feat = ti.m * BM + q * 32 + lane;     // output feature of this thread
      if (GATED) {
        // h = silu(g) * u; one e4m3 scale per (row, the tile's 128 features)
        float* red_p = red + (tiles_done & 1) * 4 * BN;          // [q][column]
#pragma unroll
        for (int c = 0; c < C::COLS; ++c) {
          const float g = acc_g[c];
          const float h = g / (1.0f + __expf(-g)) * acc_u[c];
          acc_g[c] = h;
          float a = fabsf(h);
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
          if (lane == 0) red_p[q * BN + c0 + c] = a;
        }
        named_bar_sync(1 + cq, 128);
        if (ok) {
          uint8_t* hq = static_cast<uint8_t*>(p.d);
#pragma unroll
          for (int c = 0; c < C::COLS; ++c) {
            if (c < ncols && c0 + c < ti.nrows) {
              const float amax = fmaxf(fmaxf(red_p[0 * BN + c0 + c], red_p[1 * BN + c0 + c]),
                                       fmaxf(red_p[2 * BN + c0 + c], red_p[3 * BN + c0 + c]));
              const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
              const int row = ti.row0 + c0 + c;
              hq[(size_t)row * p.ldd + feat] = e4m3_of(__fdiv_rn(acc_g[c], s));
              if (q == 0 && lane == 0) p.sd[(size_t)ti.m * p.R_cap + row] = s;
            }
          }
        }
      } else if (ok) {
        __nv_bfloat16* y = static_cast<__nv_bfloat16*>(p.d);
#pragma unroll
        for (int c = 0; c < C::COLS; ++c)
          if (c < ncols && c0 + c < ti.nrows)
            y[(size_t)(ti.row0 + c0 + c) * p.ldd + feat] = __float2bfloat16_rn(acc_g[c]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encoder8() {
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

// Row-major byte matrix [outer, inner] read in boxes of box_outer rows x 128
// bytes, 128-byte swizzle, zero fill out of bounds.
bool make_map_u8(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
                 uint32_t box_outer) {
  auto enc = encoder8();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t prepare_grouped_gemm_fp8_kernels() {
  cudaError_t e = cudaFuncSetAttribute(grouped_gemm_fp8_kernel<true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Cfg8<true>::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(grouped_gemm_fp8_kernel<false>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              Cfg8<false>::SMEM_BYTES);
}

cudaError_t launch_grouped_gemm_fp8(const GroupedGemmFp8Args& a, cudaStream_t st) {
  CUtensorMap tmA, tmAs, tmB;
  const uint64_t rows_routed = (uint64_t)a.E * a.rows_per_expert;
  if (!make_map_u8(&tmA, a.a_routed, a.K_routed, rows_routed, BM)) return cudaErrorInvalidValue;
  if (a.a_shared != nullptr) {
    const uint64_t rows_shared = (uint64_t)a.m_tiles_shared * BM * (a.gated ? 2 : 1);
    if (!make_map_u8(&tmAs, a.a_shared, a.K_shared, rows_shared, BM))
      return cudaErrorInvalidValue;
  } else {
    tmAs = tmA;
  }
  if (!make_map_u8(&tmB, a.b, a.K_ld, (uint64_t)a.R_cap, 16)) return cudaErrorInvalidValue;

  KParams8 p;
  p.group_offsets = a.group_offsets;
  p.E = a.E;
  p.G = a.G;
  p.kb_routed = a.K_routed / BK;
  p.kb_shared = a.K_shared / BK;
  p.rows_per_expert = a.rows_per_expert;
  p.m_routed = a.m_tiles_routed;
  p.m_shared = a.m_tiles_shared;
  p.up_routed = a.up_routed;
  p.up_shared = a.up_shared;
  p.sa_routed = a.sa_routed;
  p.sa_shared = a.sa_shared != nullptr ? a.sa_shared : a.sa_routed;
  p.sb = a.sb;
  p.d = a.d;
  p.sd = a.sd;
  p.ldd = a.ldd;
  p.R_cap = a.R_cap;
  p.status = a.status;
  p.timeout_bit = a.timeout_bit;
  p.wait_limit_ns = a.wait_limit_ns;
  if (a.gated) {
    grouped_gemm_fp8_kernel<true><<<a.num_ctas, kThreads, Cfg8<true>::SMEM_BYTES, st>>>(
        tmA, tmAs, tmB, p);
  } else {
    grouped_gemm_fp8_kernel<false><<<a.num_ctas, kThreads, Cfg8<false>::SMEM_BYTES, st>>>(
        tmA, tmAs, tmB, p);
  }
  return cudaGetLastError();
}

}  // namespace moe
