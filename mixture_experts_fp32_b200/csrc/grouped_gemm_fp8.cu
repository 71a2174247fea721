// Grouped expert GEMMs with e4m3 operands and fp32 block scales on tcgen05.
//
// The mixed BF16 / FP8 block-scale arithmetic of the pages (Step3 推論最適化
// (MI308X vs H20), §最適化技術; "GEMM à l'échelle bloc", AMD Instinct MI355X :
// ATOM, kernels fusionnés et montée en charge, introduction): weights carry one
// fp32 scale per 128x128 block, activations one per 1x128 group, so
//
//   acc[t, n] = sum_kb  s_a[t, kb] * s_w[n/128, kb] * sum_{k in kb} qa[t, k] * qw[n, k].
//
// The scale changes every 128 K, and arbitrary fp32 scales cannot be given to
// the tensor core's block-scaled kinds (they take power-of-two scales), so each
// 128-wide K block is multiplied (kind::f8f6f4, exact products, fp32 sums) into
// a fresh tensor-memory partial, and the epilogue warps fold every partial into
// fp32 register accumulators with its scale ("promotion").  Two partial
// buffers let the tensor core run one K block ahead of the promotion.
//
// One CTA per tile of 128 activation rows x 256 weight rows (M = 128, N = 256).
// Two things bound this loop.  The larger is the operand feed: 48 KB of shared
// memory per K block per CTA (a build of the same tile that accumulates all K
// blocks in one buffer, i.e. without promotion, still runs at about 60 % of
// the e4m3 rate on the 8192-token, 256-expert prefill).  The other is the
// hand-off of the two partial buffers: with a new scale every 128 K, tensor
// memory (512 columns) holds two K blocks of partials, and an MMA into a buffer
// must wait until the promotion has read it (about a fifth of the time on that
// workload).  Tiles of 256 rows on CTA pairs (cta_group::2, half the weight tile
// staged per CTA) read less per K block but keep the hand-off and pad groups to
// 256 rows; measured on the same prefill they were slower than this one-CTA form.
//
// Rows of activations take the MMA's M side and weight rows its N side: a TMEM
// lane is one activation row, so the activation scale of a K block is one
// register per thread and the weight scale one per 128 columns; promotion is
// one FMA per value, and each thread writes its row contiguously.
//
//   gated: a tile owns 128 features of h: the B operand stacks the matching
//          128 gate rows and 128 up rows (N = 256), so g and u of a feature sit
//          in the same TMEM lane.  After the last K block h = silu(g) * u is
//          quantised per 1x128 group (the tile's 128 features are one group)
//          into e4m3 codes and an fp32 scale.
//   down:  a tile owns up to 256 output features (two weight scale blocks); y
//          is written in bf16, each warp's rows passing through shared memory in
//          rounds of 8 so that every store covers two whole 256-byte row segments
//          (one row per thread would make every store touch 32 rows: 8-12 % of the
//          down GEMM's time on the 8192-token prefill).
//
// Signalled sends (down GEMM of an expert-parallel rank): a cooperative launch
// whose first n_gemm CTAs run the tiles, every epilogue warp counting each stored
// tile in its group's counter, while the other CTAs copy each finished group's
// rows to the owners' slabs.
//
// Three warpgroups (384 threads).  Warpgroup 0: warp 0 issues TMA loads, warp 1
// owns tensor memory and issues the MMAs; it gives registers back
// (setmaxnreg.dec).  Warpgroups 1 and 2 (8 warps) promote and finish, with the
// registers warpgroup 0 released: warp w reads TMEM lanes 32*(w%4)... and one
// half of the tile's columns, 128 fp32 accumulators a thread.  Every wait is
// bounded; the two on the partial-buffer hand-off (the MMA issuer's for a free
// buffer, the epilogue's for a written one) poll instead of suspending, the others
// suspend.
#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int BMT = 128;           // activation rows per tile (MMA M)
constexpr int BK = 128;            // e4m3 elements (= bytes) per K block: one scale group
constexpr int BNW = 256;           // weight rows per tile (MMA N)
constexpr int kEpiWarps = 8;       // two per TMEM lane quadrant, each half of the columns
constexpr int kThreads = 384;
// 12 warps leave each SM sub-partition three warps: 168 registers a thread at
// launch.  Warpgroup 0 drops to 56, warpgroups 1-2 rise to 224:
// 128 * 56 + 256 * 224 = 384 * 168 = 64512 registers, and per sub-partition
// 56 + 224 + 224 = 504 <= 512.
constexpr int kLaunchRegs = 168;
constexpr int kProducerRegs = 56;
constexpr int kEpilogueRegs = 224;
static_assert(128 * kProducerRegs + 256 * kEpilogueRegs == kThreads * kLaunchRegs,
              "register shares must add up to the launch's registers");
constexpr uint32_t kTmemCols = 512;
constexpr int kPartStride = 256;   // TMEM columns between the two partial buffers
constexpr int A_BYTES = BMT * BK;              // 16 KB: the tile's activation rows
constexpr int B_BYTES = BNW * BK;              // 32 KB: all 256 weight rows
constexpr int STAGES = 4;
constexpr int DATA_BYTES = STAGES * (A_BYTES + B_BYTES);
constexpr int RED_BYTES = 2 * BMT * 2 * 4;    // h amax halves [tile parity][row][half]
constexpr int kGroupSlots = kMaxExperts + 4;   // >= groups + 1
// down: y rows staged per warp, 8 rows x 256 bytes, so that stores cover whole rows
// (the gated kernel has no staging, which leaves it more L1)
constexpr int STG_BYTES = kEpiWarps * 8 * 256;
template <bool GATED>
constexpr int smem_bytes() {
  return DATA_BYTES + RED_BYTES + (GATED ? 0 : STG_BYTES) + 1024 + 256 + 2 * 4 * kGroupSlots;
}
static_assert(smem_bytes<false>() <= 227 * 1024, "shared memory of one CTA");
constexpr unsigned long long kTeardownLimitNs = 1000000000ull;

// A scale fetched ahead of its use: the asm keeps the load where it is written
// (the compiler may not sink it next to the use and expose its latency).
__device__ __forceinline__ float ldg_ahead(const float* p) {
  float v;
  asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}

// Two 16-column TMEM loads without a wait, and the wait that ties the
// registers of two such pairs: no use of r or q can be scheduled before it.
__device__ __forceinline__ void tmem_ld_2x16(uint32_t a0, uint32_t a1, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%32];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%16, %17, %18, %19, %20, %21, %22, %23, %24, "
      "%25, %26, %27, %28, %29, %30, %31}, [%33];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(a0), "r"(a1)
      : "memory");
}

__device__ __forceinline__ void tmem_ld_wait_tied2(uint32_t (&r)[32], uint32_t (&q)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                 "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31]), "+r"(q[0]), "+r"(q[1]), "+r"(q[2]), "+r"(q[3]),
                 "+r"(q[4]), "+r"(q[5]), "+r"(q[6]), "+r"(q[7]), "+r"(q[8]), "+r"(q[9]),
                 "+r"(q[10]), "+r"(q[11]), "+r"(q[12]), "+r"(q[13]), "+r"(q[14]), "+r"(q[15]),
                 "+r"(q[16]), "+r"(q[17]), "+r"(q[18]), "+r"(q[19]), "+r"(q[20]), "+r"(q[21]),
                 "+r"(q[22]), "+r"(q[23]), "+r"(q[24]), "+r"(q[25]), "+r"(q[26]), "+r"(q[27]),
                 "+r"(q[28]), "+r"(q[29]), "+r"(q[30]), "+r"(q[31])
               :
               : "memory");
}

// acc[base .. base+15] += s * (32 loaded columns, as 16 pairs)
__device__ __forceinline__ void promote16(float2 (&acc)[32], int base, const uint32_t (&r)[32],
                                          float2 s) {
#pragma unroll
  for (int c = 0; c < 16; ++c)
    acc[base + c] = __ffma2_rn(make_float2(__uint_as_float(r[2 * c]), __uint_as_float(r[2 * c + 1])),
                               s, acc[base + c]);
}

struct KParams8 {
  const int* group_offsets;
  int E, G;
  int e_base;                     // the routed weights and scales start at expert e_base
  int kb_routed, kb_shared;
  int rows_per_expert;            // weight rows of one routed expert
  int ft_routed, ft_shared;       // feature tiles per group
  int feat_routed, feat_shared;   // features per group (down: H; gated: I or Is)
  int up_routed, up_shared;       // gated: row offset of the up half
  const float* sw_routed;         // [E, rows_per_expert/128, kb_routed]
  const float* sw_shared;         // [rows_shared/128, kb_shared]
  const float* sa;                // activation scales [R_cap, sa_ld] (row-major)
  int sa_ld;
  void* d;                        // gated: e4m3 h [R_cap, ldd]; down: bf16 y [R_cap, ldd]
  float* sd;                      // gated: h scales [R_cap, ldd/128]
  int ldd;
  unsigned int* status;
  unsigned int timeout_bit;
  unsigned long long wait_limit_ns;
  int n_gemm;                     // CTAs that run tiles (the rest send)
  SendArgs send;
};

struct Tile8 {
  int g, f0, nfeat, row0, nrows, k_blocks, row_tiles;
};

template <bool GATED>
__device__ __forceinline__ Tile8 decode_tile8(int t, const int* ts, const int* go,
                                              const KParams8& p) {
  int lo = 0, hi = p.G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (ts[mid] <= t) lo = mid; else hi = mid;
  }
  Tile8 ti;
  ti.g = lo;
  const bool routed = lo < p.E;
  const int gbeg = go[lo], gend = go[lo + 1];
  const int rt = (gend - gbeg + BMT - 1) / BMT;
  const int local = t - ts[lo];
  const int f = local / rt;                    // feature tile outer, row tile inner
  const int r = local - f * rt;
  const int fpt = GATED ? 128 : BNW;           // features per tile
  const int feats = routed ? p.feat_routed : p.feat_shared;
  ti.f0 = f * fpt;
  ti.nfeat = min(fpt, feats - ti.f0);
  ti.row0 = gbeg + r * BMT;
  ti.nrows = min(BMT, gend - ti.row0);
  ti.k_blocks = routed ? p.kb_routed : p.kb_shared;
  ti.row_tiles = rt;
  return ti;
}

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

template <bool GATED>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_fp8_kernel(const __grid_constant__ CUtensorMap tmA,    // activation rows
                            const __grid_constant__ CUtensorMap tmW,    // routed weights
                            const __grid_constant__ CUtensorMap tmWs,   // shared weights
                            const KParams8 p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* a_smem = base;
  uint8_t* b_smem = base + STAGES * A_BYTES;
  float* red = reinterpret_cast<float*>(base + DATA_BYTES);
  uint8_t* stg_all = base + DATA_BYTES + RED_BYTES;
  uint64_t* bars =
      reinterpret_cast<uint64_t*>(base + DATA_BYTES + RED_BYTES + (GATED ? 0 : STG_BYTES));
  uint64_t* full = bars;                 // stage loaded (TMA bytes)
  uint64_t* empty = bars + STAGES;       // stage consumed by the MMAs
  uint64_t* pfull = bars + 2 * STAGES;   // partial buffer written
  uint64_t* pempty = pfull + 2;          // partial buffer read by all epilogue warps
  uint64_t* teardown = pempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(teardown + 1);
  int* ts = reinterpret_cast<int*>(tmem_holder + 1);   // first tile of each group
  int* gos = ts + kGroupSlots;                            // group row offsets, staged

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int* go = gos;
  const int cta = blockIdx.x, nctas = p.n_gemm;
  const bool sender = !GATED && p.send.n_send > 0 && cta >= p.n_gemm;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
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
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmWs);
  }
  if (warp == 1 && !sender) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 2) {
    // tile prefix over groups: ceil(rows / 128) row tiles x feature tiles
    int running = 0;
    for (int b0 = 0; b0 < p.G; b0 += 32) {
      const int g = b0 + lane;
      int cnt = 0;
      if (g < p.G) {
        const int beg = p.group_offsets[g], end = p.group_offsets[g + 1];
        gos[g] = beg;
        const int rows = end - beg;
        cnt = (g < p.E ? p.ft_routed : p.ft_shared) * ((rows + BMT - 1) / BMT);
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
    if (lane == 0) {
      ts[p.G] = running;
      gos[p.G] = p.group_offsets[p.G];
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int total = ts[p.G];
  if (sender) {
    // 8 epilogue warps count every tile; y rows are bf16
    send_finished_groups<__nv_bfloat16>(p.send, static_cast<const __nv_bfloat16*>(p.d), p.ldd,
                                        go, ts, p.G, p.E, (unsigned int)kEpiWarps,
                                        cta - p.n_gemm, p.status, p.wait_limit_ns,
                                        reinterpret_cast<int*>(tmem_holder));
    return;
  }
  const uint32_t tmem_base = *tmem_holder;

  if (warp < 4) {
    regs_dec<kProducerRegs>();
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------- TMA producer
      // A group with one row tile reads its weights once (evict first) and its
      // rows once per feature tile (evict last); larger groups reuse both from
      // L2 across neighbouring tiles (evict normal).
      const uint64_t pol_first = policy_evict_first();
      const uint64_t pol_last = policy_evict_last();
      const uint64_t pol_normal = policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0, issued = 0, parity = 0;
      bool ok = true;
      for (int t = cta; t < total && ok; t += nctas) {
        const Tile8 ti = decode_tile8<GATED>(t, ts, go, p);
        const bool routed = ti.g < p.E;
        const CUtensorMap* wm = routed ? &tmW : &tmWs;
        const int wrow = (routed ? (ti.g - p.e_base) * p.rows_per_expert : 0) + ti.f0;
        const int up = routed ? p.up_routed : p.up_shared;
        const int brow0 = wrow, brow1 = GATED ? wrow + up : wrow + 128;
        const int arow = ti.row0;
        const uint64_t pol_a = ti.row_tiles == 1 ? pol_last : pol_normal;
        const uint64_t pol_w = ti.row_tiles == 1 ? pol_first : pol_normal;
        for (int kb = 0; kb < ti.k_blocks; ++kb) {
          if (!mbar_wait_sleep(smem_u32(&empty[stage]), phase ^ 1u, p.wait_limit_ns, p.status,
                               p.timeout_bit)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_arrive_expect_tx(fb, A_BYTES + B_BYTES);
          tma_load_2d(smem_u32(a_smem + stage * A_BYTES), &tmA, kb * BK, arow, fb, pol_a);
          tma_load_2d(smem_u32(b_smem + stage * B_BYTES), wm, kb * BK, brow0, fb, pol_w);
          tma_load_2d(smem_u32(b_smem + stage * B_BYTES + 128 * BK), wm, kb * BK, brow1, fb, pol_w);
          issued |= 1u << stage;
          parity = (parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // no load may still be writing when the CTA leaves: wait until the MMAs
      // have consumed the last load of every stage (which follows its arrival)
      for (int s = 0; s < STAGES; ++s)
        if ((issued >> s) & 1u)
          mbar_wait_sleep(smem_u32(&empty[s]), (parity >> s) & 1u, kTeardownLimitNs, p.status,
                          p.timeout_bit);
    } else if (warp == 1 && lane == 0) {
      // ----------------------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t kcount = 0;          // K blocks issued so far: partial buffer = kcount & 1
      bool ok = true, any = false;
      for (int t = cta; t < total && ok; t += nctas) {
        const int k_blocks = decode_tile8<GATED>(t, ts, go, p).k_blocks;
        for (int kb = 0; kb < k_blocks; ++kb, ++kcount) {
          const uint32_t pb = kcount & 1u;
          const uint32_t use = kcount >> 1;
          if (!mbar_wait_bounded(smem_u32(&pempty[pb]), (use & 1u) ^ 1u, p.wait_limit_ns,
                                 p.status, p.timeout_bit) ||
              !mbar_wait_sleep(smem_u32(&full[stage]), phase, p.wait_limit_ns, p.status,
                               p.timeout_bit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d0 = tmem_base + pb * kPartStride;
          const uint64_t a_desc = smem_desc_sw128(smem_u32(a_smem + stage * A_BYTES));
          const uint64_t b_desc = smem_desc_sw128(smem_u32(b_smem + stage * B_BYTES));
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)   // +32 bytes per K step = 2 in the address field
            umma_e4m3(d0, a_desc + 2 * kk, b_desc + 2 * kk, idesc_e4m3_m128(BNW), kk != 0);
          umma_commit(smem_u32(&empty[stage]));
          umma_commit(smem_u32(&pfull[pb]));
          any = true;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (any) {
        umma_commit(smem_u32(teardown));
        mbar_wait_sleep(smem_u32(teardown), 0, kTeardownLimitNs, p.status, p.timeout_bit);
      }
    }
    __syncwarp();
  } else {
    regs_inc<kEpilogueRegs>();
    // ------------------------------------------------- promotion and epilogue
    // Thread = one activation row of the tile (its TMEM lane) and one half of
    // the tile's columns.  Every epilogue warp walks the
    // same tiles and K blocks and, for gated tiles, passes one named barrier
    // per tile whatever happens: after an expired wait it keeps walking
    // without further waits, loads or stores.  Rows past the group's end are
    // computed by the MMA but neither promoted nor stored.
    const int ew = warp - 4;              // 0..7
    const int q = warp & 3;               // TMEM lane quadrant
    const int hh = ew >> 2;               // column half
    const int r = q * 32 + lane;          // row within this CTA's 128
    // Per-tile state of this thread; the next tile's is set up (and its first
    // scales requested) before the current tile's finishing work, so that the
    // loads' latency hides behind it.
    struct EpiTile {
      int g, row0, rows, f0, nfeat, k_blocks;
      const float* sa_row;
      const float* swa;
      const float* swb;
    };
    auto setup = [&](int t, EpiTile& e, float& a0, float& wa0, float& wb0) {
      const Tile8 ti = decode_tile8<GATED>(t, ts, go, p);
      const bool routed = ti.g < p.E;
      e.g = ti.g;
      e.row0 = ti.row0;
      e.rows = ti.nrows;
      e.f0 = ti.f0;
      e.nfeat = ti.nfeat;
      e.k_blocks = ti.k_blocks;
      const float* sw = routed ? p.sw_routed + (size_t)(ti.g - p.e_base) *
                                                   (p.rows_per_expert / 128) * ti.k_blocks
                               : p.sw_shared;
      // weight scale rows: gated -> gate block and up block of f0; down -> block of this half
      const int up = routed ? p.up_routed : p.up_shared;
      // (down: a half past a partial last tile reads its tile's last block, in bounds)
      e.swa = sw + (size_t)((GATED ? ti.f0 : min(ti.f0 + hh * 128, ti.f0 + ti.nfeat - 1)) / 128) *
                       ti.k_blocks;
      e.swb = sw + (size_t)((up + ti.f0) / 128) * ti.k_blocks;
      // rows past the group read the tile's first row instead (in bounds, unused)
      e.sa_row = p.sa + (size_t)(r < e.rows ? e.row0 + r : ti.row0) * p.sa_ld;
      a0 = ldg_ahead(e.sa_row);
      wa0 = ldg_ahead(e.swa);
      wb0 = GATED ? ldg_ahead(e.swb) : 0.f;
    };
    uint32_t kcount = 0;
    int tiles_done = 0;
    bool ok = true;
    EpiTile cur;
    float nxt_a = 0.f, nxt_wa = 0.f, nxt_wb = 0.f;
    if (cta < total) setup(cta, cur, nxt_a, nxt_wa, nxt_wb);
    for (int t = cta; t < total; t += nctas, ++tiles_done) {
      const bool live = r < cur.rows;
      const bool warp_live = q * 32 < cur.rows;
      const bool any_cols = GATED || hh * 128 < cur.nfeat;

      // gated: g and u of 64 features; down: 128 features.  Pairs of columns
      // are updated by one packed fp32 FMA (same rounding as two scalar FMAs).
      float2 acc_a[32], acc_b[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        acc_a[c] = make_float2(0.f, 0.f);
        acc_b[c] = make_float2(0.f, 0.f);
      }
      for (int kb = 0; kb < cur.k_blocks; ++kb, ++kcount) {
        const uint32_t pb = kcount & 1u;
        const uint32_t use = kcount >> 1;
        const float sa_cur = live ? nxt_a : 0.f;
        const float s_a = nxt_wa * sa_cur;
        const float s_b = (GATED ? nxt_wb : nxt_wa) * sa_cur;
        if (kb + 1 < cur.k_blocks) {                  // next block's factors, fetched early
          nxt_a = ldg_ahead(cur.sa_row + kb + 1);
          nxt_wa = ldg_ahead(cur.swa + kb + 1);
          if (GATED) nxt_wb = ldg_ahead(cur.swb + kb + 1);
        }
        if (ok)
          ok = mbar_wait_bounded_warp(smem_u32(&pfull[pb]), use & 1u, p.wait_limit_ns,
                                      p.status, p.timeout_bit);
        if (!ok) continue;
        tc_fence_after();
        // the partial buffer goes back to the MMA issuer as soon as it has been read
        auto release = [&]() {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&pempty[pb]));
        };
        if (any_cols && warp_live) {
          const uint32_t tl = tmem_base + ((uint32_t)(q * 32) << 16) + pb * kPartStride;
          const float2 sa2 = make_float2(s_a, s_a), sb2 = make_float2(s_b, s_b);
          uint32_t ra[32], rb[32];
          // gated: gate columns hh*64 .. +63 -> acc_a, up columns 128 + hh*64 .. -> acc_b;
          // down: columns hh*128 .. +63 -> acc_a, +64 .. +127 -> acc_b (one scale block).
          // Two TMEM round trips of 64 columns; the buffer is released after the second
          // (the last 32 FMAs after the release).
          const uint32_t c0 = GATED ? tl + hh * 64 : tl + hh * 128;
          const uint32_t c1 = GATED ? tl + 128 + hh * 64 : tl + hh * 128 + 64;
          tmem_ld_2x16(c0, c0 + 16, ra);
          tmem_ld_2x16(c1, c1 + 16, rb);
          tmem_ld_wait_tied2(ra, rb);
          promote16(acc_a, 0, ra, sa2);
          promote16(acc_b, 0, rb, sb2);
          tmem_ld_2x16(c0 + 32, c0 + 48, ra);
          tmem_ld_2x16(c1 + 32, c1 + 48, rb);
          tmem_ld_wait_tied2(ra, rb);
          release();
          promote16(acc_a, 16, ra, sa2);
          promote16(acc_b, 16, rb, sb2);
        } else {
          release();
        }
      }

      const EpiTile fin = cur;                       // the tile being finished
      if (t + nctas < total) setup(t + nctas, cur, nxt_a, nxt_wa, nxt_wb);

      if (GATED) {
        // h = silu(g) * u over this thread's 64 features; the row's scale needs
        // the max over both halves (the partner warp holds the other 64).
        // silu's quotient uses the fast reciprocal division (about 2 ulp; its
        // denominator 1 + e^-g is >= 1 and saturates to +inf, giving -0 for
        // g -> -inf): h is quantised to 3 mantissa bits right after.
        float amax = 0.f;
        float hv[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float g = (c & 1) ? acc_a[c >> 1].y : acc_a[c >> 1].x;
          const float u = (c & 1) ? acc_b[c >> 1].y : acc_b[c >> 1].x;
          hv[c] = __fdividef(g, 1.0f + __expf(-g)) * u;
          amax = fmaxf(amax, fabsf(hv[c]));
        }
        float* red_p = red + (tiles_done & 1) * BMT * 2;
        red_p[r * 2 + hh] = amax;
        named_bar_sync(1, kEpiWarps * 32);
        if (ok && live) {
          const float m = fmaxf(red_p[r * 2], red_p[r * 2 + 1]);
          const float s = m > 0.f ? __fdiv_rn(m, 448.f) : 1.f;
          // codes: h * (1/s) rounded to e4m3, the reciprocal once per row
          const float inv = __frcp_rn(s);
          const int row = fin.row0 + r;
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.d) + (size_t)row * p.ldd +
                                                fin.f0 + hh * 64);
#pragma unroll
          for (int w4 = 0; w4 < 4; ++w4) {
            uint4 o;
            uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int c = w4 * 16 + j * 4;
              ow[j] = e4m3x4(hv[c] * inv, hv[c + 1] * inv, hv[c + 2] * inv, hv[c + 3] * inv);
            }
            dst[w4] = o;
          }
          if (hh == 0) p.sd[(size_t)row * (p.ldd / 128) + fin.f0 / 128] = s;
        }
      } else if (ok && any_cols) {
        // bf16 y: this warp's 32 rows x 128 columns go out in four rounds of 8 rows.
        // The round's 8 lanes put their 256-byte row segments into shared memory
        // (16-byte chunk c of row j at slot c ^ j: no bank conflicts either way),
        // then every store instruction writes two whole segments (lanes 0-15 one row,
        // 16-31 the next), so that the stores cover whole cache lines.
        uint8_t* stg = stg_all + ew * (8 * 256);
        const uint32_t stg_s = smem_u32(stg);
        const int wrow = q * 32;                         // this warp's first row in the tile
        uint32_t pk[64];                                 // the row's 128 bf16, packed in pairs
#pragma unroll
        for (int c2 = 0; c2 < 64; ++c2) {
          const float2 a = c2 < 32 ? acc_a[c2] : acc_b[c2 - 32];
          const __nv_bfloat162 b = __floats2bfloat162_rn(a.x, a.y);
          pk[c2] = *reinterpret_cast<const uint32_t*>(&b);
        }
#pragma unroll 1
        for (int rnd = 0; rnd < 4; ++rnd) {
          if ((lane >> 3) == rnd) {
            const int j = lane & 7;
#pragma unroll
            for (int w8 = 0; w8 < 16; ++w8)
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                               stg_s + j * 256 + ((w8 ^ j) & 15) * 16),
                           "r"(pk[4 * w8]), "r"(pk[4 * w8 + 1]), "r"(pk[4 * w8 + 2]),
                           "r"(pk[4 * w8 + 3])
                           : "memory");
          }
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int j = 2 * i + (lane >> 4);           // row within the round
            const int c = lane & 15;                     // 16-byte chunk of the segment
            uint4 o;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(o.x), "=r"(o.y), "=r"(o.z), "=r"(o.w)
                         : "r"(stg_s + j * 256 + ((c ^ j) & 15) * 16)
                         : "memory");
            const int tr = wrow + rnd * 8 + j;           // row within the tile
            if (tr < fin.rows) {
              __nv_bfloat16* y = static_cast<__nv_bfloat16*>(p.d) +
                                 (size_t)(fin.row0 + tr) * p.ldd + fin.f0 + hh * 128;
              reinterpret_cast<uint4*>(y)[c] = o;
            }
          }
          __syncwarp();
        }
      }
      if (!GATED && p.send.n_send > 0) signal_tile_stored(p.send.done, fin.g);
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

// Row-major byte matrix [outer, inner] read in boxes of 128 rows x 128 bytes,
// 128-byte swizzle, zero fill out of bounds.
bool make_map_u8(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer) {
  auto enc = encoder8();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {(cuuint32_t)BK, 128};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The register shares of the warpgroups only add up if the kernel was built
// with exactly kLaunchRegs registers a thread; anything else is refused rather
// than launched (a mismatched split would wait forever).
template <bool GATED>
cudaError_t check_register_split() {
  cudaFuncAttributes attr;
  cudaError_t e = cudaFuncGetAttributes(&attr, grouped_gemm_fp8_kernel<GATED>);
  if (e != cudaSuccess) return e;
  return attr.numRegs == kLaunchRegs ? cudaSuccess : cudaErrorInvalidConfiguration;
}

}  // namespace

cudaError_t prepare_grouped_gemm_fp8_kernels() {
  cudaError_t e = check_register_split<true>();
  if (e == cudaSuccess) e = check_register_split<false>();
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(grouped_gemm_fp8_kernel<true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes<true>());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(grouped_gemm_fp8_kernel<false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes<false>());
  return e;
}

cudaError_t launch_grouped_gemm_fp8(const GroupedGemmFp8Args& a, cudaStream_t st) {
  CUtensorMap tmA, tmW, tmWs;
  if (!make_map_u8(&tmA, a.b, a.K_ld, (uint64_t)a.R_cap)) return cudaErrorInvalidValue;
  const uint64_t rows_routed = (uint64_t)a.n_local * a.rows_per_expert;
  if (!make_map_u8(&tmW, a.a_routed, a.K_routed, rows_routed)) return cudaErrorInvalidValue;
  if (a.a_shared != nullptr) {
    const uint64_t rows_shared = a.gated ? (uint64_t)2 * a.up_shared : (uint64_t)a.feat_shared;
    if (!make_map_u8(&tmWs, a.a_shared, a.K_shared, rows_shared)) return cudaErrorInvalidValue;
  } else {
    tmWs = tmW;
  }

  KParams8 p;
  p.group_offsets = a.group_offsets;
  p.E = a.E;
  p.G = a.G;
  p.e_base = a.e_base;
  p.kb_routed = a.K_routed / BK;
  p.kb_shared = a.K_shared / BK;
  p.rows_per_expert = a.rows_per_expert;
  const int fpt = a.gated ? 128 : BNW;
  p.feat_routed = a.feat_routed;
  p.feat_shared = a.feat_shared;
  p.ft_routed = (a.feat_routed + fpt - 1) / fpt;
  p.ft_shared = (a.feat_shared + fpt - 1) / fpt;
  p.up_routed = a.up_routed;
  p.up_shared = a.up_shared;
  p.sw_routed = a.sa_routed;
  p.sw_shared = a.sa_shared != nullptr ? a.sa_shared : a.sa_routed;
  p.sa = a.sb;
  p.sa_ld = a.K_ld / BK;
  p.d = a.d;
  p.sd = a.sd;
  p.ldd = a.ldd;
  p.status = a.status;
  p.timeout_bit = a.timeout_bit;
  p.wait_limit_ns = a.wait_limit_ns;
  p.send = a.send;
  if (a.gated) p.send.n_send = 0;
  p.n_gemm = a.num_ctas - p.send.n_send;
  if (p.n_gemm < 1) return cudaErrorInvalidValue;

  if (a.gated) {
    grouped_gemm_fp8_kernel<true><<<a.num_ctas, kThreads, smem_bytes<true>(), st>>>(tmA, tmW, tmWs,
                                                                                    p);
  } else if (p.send.n_send == 0) {
    grouped_gemm_fp8_kernel<false><<<a.num_ctas, kThreads, smem_bytes<false>(), st>>>(tmA, tmW,
                                                                                      tmWs, p);
  } else {
    // the senders wait on the tiles: every CTA must be resident at once
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.num_ctas, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes<false>();
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, grouped_gemm_fp8_kernel<false>, tmA, tmW, tmWs, p);
  }
  return cudaGetLastError();
}

}  // namespace moe
