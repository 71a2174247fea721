// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05, TMEM
// accumulators, TMA-fed shared-memory ring), persistent, one CTA per SM.
//
// The expert FFN of an MoE layer (Step3 推論最適化 (MI308X vs H20), §最適化技術:
// a one-stage MoE kernel tuned along inter_dim, the shared-expert MLP fused
// into the layer; [SGLang] MoE 모델을 위한 Single Batch Overlap 기법, §들어가며:
// the down projection GEMM) runs as two launches of this kernel:
//
//   gated (gate/up):  h[r, i] = silu(g) * u,  g = Wg[e][i,:] . x_perm[r,:],
//                                              u = Wu[e][i,:] . x_perm[r,:]
//   down:             y[r, o] = Wd[e][o,:] . h[r,:]     (kept in fp32 for the combine)
//
// h leaves the gated epilogue in two bf16 parts, hi = bf16(h) and lo = bf16(h - hi),
// stored as rows 2r and 2r + 1 of the h buffer, and the down GEMM multiplies both
// (2N rows on the MMA's N side) and adds the two columns of a row in fp32: the
// tensor core takes bf16 operands, and the two parts carry h to 16 significant
// bits instead of 8, so rounding h no longer shows in the layer's output (with
// hi alone it cost up to about half a percent of the output rms, which with the
// output's own bf16 rounding came close to the 2 % bound).  The down GEMM takes
// at most 96 rows a tile, so that a tile's 2 x 96 part rows fit one 192-row box.
//
// for every permuted row r of group e (routed experts, then the shared one).
// Decode batches give each expert only a handful of rows, so the weights take
// the MMA's M side (128 weight rows per tile) and the rows take N (16..128,
// rounded up to 16): the weight stream, which dominates HBM traffic, is read
// once, in 128x64 TMA boxes.  SwiGLU is fused into the gated epilogue: a tile
// owns 128 gate rows and the matching 128 up rows, accumulated side by side in
// tensor memory, so each epilogue thread holds g and u for the same i.
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 owns tensor memory
// and issues the MMAs, warps 2-5 drain the accumulators (warp w reads TMEM
// lanes 32*(w%4)...).  Two accumulator buffers let the epilogue of one tile
// overlap the main loop of the next.  Tiles are enumerated on the device from
// the group offsets (no host round trip), and every CTA walks tiles
// blockIdx.x, blockIdx.x + gridDim.x, ...  Every wait is bounded.
//
// Signalled sends (down GEMM of an expert-parallel rank): the launch is
// cooperative (all CTAs resident), its first n_gemm CTAs run the tiles as above
// and every epilogue warp counts each stored tile in its group's counter; the
// other CTAs copy each group's rows to the owners' slabs as soon as the group's
// count is complete, while later groups are still being multiplied.
#include <cudaTypedefs.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int BM = 128;            // weight rows per MMA
constexpr int BK = 64;             // K elements per stage (128 bytes of bf16: one swizzle row)
constexpr int BN = 128;            // max activation rows per gated tile
constexpr int BN_DOWN = 96;        // max h rows per down tile: 2 x 96 part rows per box
template <bool GATED>
__host__ __device__ constexpr int tile_rows() { return GATED ? BN : BN_DOWN; }
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr int kAccStride = 256;    // TMEM columns between the two accumulator buffers
constexpr unsigned long long kTeardownLimitNs = 1000000000ull;

template <bool GATED>
struct Cfg {
  static constexpr int A_BYTES = (GATED ? 2 : 1) * BM * BK * 2;
  // the largest B box: 128 activation rows (gated) or 2 x 96 part rows of h (down)
  static constexpr int B_ROWS = GATED ? BN : 2 * BN_DOWN;
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  // down: one weight box per stage, so more stages keep HBM bytes in flight
  // (5 x 40 KB + 3 KB of the 227 KB a CTA may have)
  static constexpr int STAGES = GATED ? 4 : 5;
  static constexpr int DATA_BYTES = STAGES * (A_BYTES + B_BYTES);
  static constexpr int SMEM_BYTES = DATA_BYTES + 1024 + 2048;
};

struct KParams {
  const int* group_offsets;
  int E, G;
  int e_base;       // the routed weights start at expert e_base
  int kb_routed, kb_shared;
  int rows_per_expert;
  int m_routed, m_shared;
  int up_routed, up_shared;
  void* d;          // gated: bf16 h rows; down: fp32 y rows
  int ldd;
  unsigned int* status;
  unsigned int timeout_bit;
  unsigned long long wait_limit_ns;
  int n_gemm;       // CTAs that run tiles (the rest send)
  SendArgs send;
};

struct Tile {
  int g, m, row0, nrows, n_mma, k_blocks;
};

template <bool GATED>
__device__ __forceinline__ Tile decode_tile(int t, const int* ts, const int* go, const KParams& p) {
  constexpr int TR = tile_rows<GATED>();
  int lo = 0, hi = p.G;   // invariant: ts[lo] <= t < ts[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (ts[mid] <= t) lo = mid; else hi = mid;
  }
  Tile ti;
  ti.g = lo;
  const int gbeg = go[lo], gend = go[lo + 1];
  const int nt = (gend - gbeg + TR - 1) / TR;
  const int local = t - ts[lo];
  ti.m = local / nt;
  const int n = local - ti.m * nt;
  ti.row0 = gbeg + n * TR;
  ti.nrows = min(TR, gend - ti.row0);
  ti.n_mma = (ti.nrows + 15) & ~15;
  ti.k_blocks = lo < p.E ? p.kb_routed : p.kb_shared;
  return ti;
}

template <bool GATED>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmAs,
                        const __grid_constant__ CUtensorMap tmB16,
                        const __grid_constant__ CUtensorMap tmB32,
                        const __grid_constant__ CUtensorMap tmB64,
                        const __grid_constant__ CUtensorMap tmB128, const KParams p) {
  using C = Cfg<GATED>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* a_smem = base;
  uint8_t* b_smem = base + C::STAGES * C::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + C::DATA_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* tfull = bars + 2 * C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* teardown = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(teardown + 1);
  int* ts = reinterpret_cast<int*>(tmem_holder + 1);   // [G + 1] tile prefix

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int* go = p.group_offsets;
  const bool sender = !GATED && p.send.n_send > 0 && (int)blockIdx.x >= p.n_gemm;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&tfull[b]), 1);
      mbar_init(smem_u32(&tempty[b]), 4);
    }
    mbar_init(smem_u32(teardown), 1);
    fence_mbarrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmAs);
    tma_prefetch_desc(&tmB16);
    tma_prefetch_desc(&tmB32);
    tma_prefetch_desc(&tmB64);
    tma_prefetch_desc(&tmB128);
  }
  if (warp == 1 && !sender) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 2) {
    // tile prefix over groups: group g has m_tiles * ceil(rows / BN) tiles
    int running = 0;
    for (int b0 = 0; b0 < p.G; b0 += 32) {
      const int g = b0 + lane;
      int cnt = 0;
      if (g < p.G) {
        const int rows = go[g + 1] - go[g];
        cnt = (g < p.E ? p.m_routed : p.m_shared) *
              ((rows + tile_rows<GATED>() - 1) / tile_rows<GATED>());
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
  const int total = ts[p.G];
  if (sender) {
    // 4 epilogue warps count every tile
    send_finished_groups<float>(p.send, static_cast<const float*>(p.d), p.ldd, go, ts, p.G, p.E,
                                4u, (int)blockIdx.x - p.n_gemm, p.status, p.wait_limit_ns,
                                reinterpret_cast<int*>(tmem_holder));
    return;
  }
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_a = policy_evict_first();
      const uint64_t pol_b = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0, issued = 0, parity = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += p.n_gemm) {
        const Tile ti = decode_tile<GATED>(t, ts, go, p);
        const bool routed = ti.g < p.E;
        const CUtensorMap* am = routed ? &tmA : &tmAs;
        const int arow = (routed ? (ti.g - p.e_base) * p.rows_per_expert : 0) + ti.m * BM;
        const int up = routed ? p.up_routed : p.up_shared;
        // the tile's rows in one box of 16/32/64/128 rows (one copy from the single
        // producer thread per K block; rows past the group come from L2 and go unused);
        // down: the h rows' two parts, 2 x n_mma rows from row 2 x row0
        // (box heights: gated 16/32/64/128, down 32/64/128/192 part rows)
        const int brows = GATED ? ti.n_mma : 2 * ti.n_mma;
        const int b0 = GATED ? 16 : 32;
        const int box = brows <= b0 ? b0 : brows <= 2 * b0 ? 2 * b0 : brows <= 4 * b0 ? 4 * b0
                      : C::B_ROWS;
        const CUtensorMap* bm =
            box == b0 ? &tmB16 : box == 2 * b0 ? &tmB32 : box == 4 * b0 ? &tmB64 : &tmB128;
        const uint32_t bytes = C::A_BYTES + box * BK * 2;
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
          if (GATED) tma_load_2d(a_dst + BM * BK * 2, am, kb * BK, arow + up, fb, pol_a);
          const uint32_t b_dst = smem_u32(b_smem + stage * C::B_BYTES);
          tma_load_2d(b_dst, bm, kb * BK, GATED ? ti.row0 : 2 * ti.row0, fb, pol_b);
          issued |= 1u << stage;
          parity = (parity & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // never leave the CTA with copies in flight
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
      bool ok = true, any = false;
      int local = 0;
      for (int t = blockIdx.x; t < total && ok; t += p.n_gemm, ++local) {
        const Tile ti = decode_tile<GATED>(t, ts, go, p);
        const int buf = local & 1;
        const uint32_t use = (uint32_t)(local >> 1);
        if (!mbar_wait_bounded(smem_u32(&tempty[buf]), (use & 1u) ^ 1u, p.wait_limit_ns, p.status,
                               p.timeout_bit)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_m128(GATED ? ti.n_mma : 2 * ti.n_mma);
        const uint32_t d_gate = tmem_base + buf * kAccStride;
        const uint32_t d_up = d_gate + BN;
        for (int kb = 0; kb < ti.k_blocks; ++kb) {
          if (!mbar_wait_bounded(smem_u32(&full[stage]), phase, p.wait_limit_ns, p.status,
                                 p.timeout_bit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a_desc = smem_desc_sw128(smem_u32(a_smem + stage * C::A_BYTES));
          const uint64_t b_desc = smem_desc_sw128(smem_u32(b_smem + stage * C::B_BYTES));
          const uint64_t au_desc =
              smem_desc_sw128(smem_u32(a_smem + stage * C::A_BYTES + BM * BK * 2));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t acc = (kb | kk) != 0;
            // +32 bytes per 16-element K step, in 16-byte units of the address field
            umma_bf16(d_gate, a_desc + 2 * kk, b_desc + 2 * kk, idesc, acc);
            if (GATED) umma_bf16(d_up, au_desc + 2 * kk, b_desc + 2 * kk, idesc, acc);
          }
          umma_commit(smem_u32(&empty[stage]));
          any = true;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(smem_u32(&tfull[buf]));
      }
      if (any) {
        // every MMA this thread issued has finished before TMEM is released
        umma_commit(smem_u32(teardown));
        mbar_wait_bounded(smem_u32(teardown), 0, kTeardownLimitNs, p.status, p.timeout_bit);
      }
    }
    __syncwarp();
  } else {
    // --------------------------------------------------------------- epilogue
    const int q = warp & 3;               // TMEM lane quadrant of this warp
    int local = 0;
    for (int t = blockIdx.x; t < total; t += p.n_gemm, ++local) {
      const Tile ti = decode_tile<GATED>(t, ts, go, p);
      const int buf = local & 1;
      const uint32_t use = (uint32_t)(local >> 1);
      if (!mbar_wait_bounded_warp(smem_u32(&tfull[buf]), use & 1u, p.wait_limit_ns, p.status,
                             p.timeout_bit))
        break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + buf * kAccStride;
      const int col = ti.m * BM + q * 32 + lane;
      const size_t dofs = (size_t)ti.row0 * p.ldd + col;
      if (GATED) {
        // h = silu(g) * u as two bf16 parts: hi in row 2r, lo = bf16(h - hi) in row 2r + 1
        __nv_bfloat16* h2 = static_cast<__nv_bfloat16*>(p.d) + (size_t)2 * ti.row0 * p.ldd + col;
        for (int c0 = 0; c0 < ti.n_mma; c0 += 16) {
          float g[16], u[16];
          tmem_ld_16(tbase + c0, g);
          tmem_ld_16(tbase + BN + c0, u);
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            if (c0 + c < ti.nrows) {
              const float h = g[c] / (1.0f + __expf(-g[c])) * u[c];
              const __nv_bfloat16 hi = __float2bfloat16_rn(h);
              const __nv_bfloat16 lo = __float2bfloat16_rn(h - __bfloat162float(hi));
              h2[(size_t)(2 * (c0 + c)) * p.ldd] = hi;
              h2[(size_t)(2 * (c0 + c) + 1) * p.ldd] = lo;
            }
          }
        }
      } else {
        // columns 2c and 2c + 1 are row c's products with hi and lo
        for (int c0 = 0; c0 < 2 * ti.n_mma; c0 += 16) {
          float v[16];
          tmem_ld_16(tbase + c0, v);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int r = c0 / 2 + c;
            if (r < ti.nrows)
              static_cast<float*>(p.d)[dofs + (size_t)r * p.ldd] = v[2 * c] + v[2 * c + 1];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty[buf]));
      if (!GATED && p.send.n_send > 0) signal_tile_stored(p.send.done, ti.g);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// Row-major bf16 matrix [outer, inner] read in boxes of box_outer rows x 64
// columns (128 bytes), 128-byte swizzle, zero fill out of bounds.
bool make_map_bf16(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
                   uint32_t box_outer) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t prepare_grouped_gemm_kernels() {
  cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Cfg<true>::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(grouped_gemm_kernel<false>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              Cfg<false>::SMEM_BYTES);
}

cudaError_t launch_grouped_gemm(const GroupedGemmArgs& a, cudaStream_t st) {
  CUtensorMap tmA, tmAs, tmB16, tmB32, tmB64, tmB128;
  const uint64_t rows_routed = (uint64_t)a.n_local * a.rows_per_expert;
  if (!make_map_bf16(&tmA, a.a_routed, a.K_routed, rows_routed, BM)) return cudaErrorInvalidValue;
  if (a.a_shared != nullptr) {
    const uint64_t rows_shared = (uint64_t)a.m_tiles_shared * BM * (a.gated ? 2 : 1);
    if (!make_map_bf16(&tmAs, a.a_shared, a.K_shared, rows_shared, BM))
      return cudaErrorInvalidValue;
  } else {
    tmAs = tmA;
  }
  // down: the h buffer holds two bf16 parts (rows 2r, 2r + 1) for each of R_cap rows,
  // read in boxes of 32/64/128/192 part rows (gated: 16/32/64/128 rows)
  const uint64_t b_rows = (uint64_t)a.R_cap * (a.gated ? 1 : 2);
  const uint32_t b0 = a.gated ? 16 : 32;
  const uint32_t b3 = a.gated ? Cfg<true>::B_ROWS : Cfg<false>::B_ROWS;
  if (!make_map_bf16(&tmB16, a.b, a.K_ld, b_rows, b0) ||
      !make_map_bf16(&tmB32, a.b, a.K_ld, b_rows, 2 * b0) ||
      !make_map_bf16(&tmB64, a.b, a.K_ld, b_rows, 4 * b0) ||
      !make_map_bf16(&tmB128, a.b, a.K_ld, b_rows, b3))
    return cudaErrorInvalidValue;

  KParams p;
  p.group_offsets = a.group_offsets;
  p.E = a.E;
  p.G = a.G;
  p.e_base = a.e_base;
  p.kb_routed = a.K_routed / BK;
  p.kb_shared = a.K_shared / BK;
  p.rows_per_expert = a.rows_per_expert;
  p.m_routed = a.m_tiles_routed;
  p.m_shared = a.m_tiles_shared;
  p.up_routed = a.up_routed;
  p.up_shared = a.up_shared;
  p.d = a.d;
  p.ldd = a.ldd;
  p.status = a.status;
  p.timeout_bit = a.timeout_bit;
  p.wait_limit_ns = a.wait_limit_ns;
  p.send = a.send;
  if (a.gated) p.send.n_send = 0;
  p.n_gemm = a.num_ctas - p.send.n_send;
  if (p.n_gemm < 1) return cudaErrorInvalidValue;
  if (a.gated) {
    grouped_gemm_kernel<true><<<a.num_ctas, kThreads, Cfg<true>::SMEM_BYTES, st>>>(
        tmA, tmAs, tmB16, tmB32, tmB64, tmB128, p);
  } else if (p.send.n_send == 0) {
    grouped_gemm_kernel<false><<<a.num_ctas, kThreads, Cfg<false>::SMEM_BYTES, st>>>(
        tmA, tmAs, tmB16, tmB32, tmB64, tmB128, p);
  } else {
    // the senders wait on the tiles: every CTA must be resident at once
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.num_ctas, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = Cfg<false>::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<false>, tmA, tmAs, tmB16, tmB32, tmB64,
                              tmB128, p);
  }
  return cudaGetLastError();
}

}  // namespace moe
