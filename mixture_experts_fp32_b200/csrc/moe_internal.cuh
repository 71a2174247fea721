// Internal declarations shared by the library's translation units: device
// helpers (mbarrier, TMA, tcgen05 in inline PTX for sm_100a) and the host-side
// launchers that the C ABI in moe_api.cu sequences.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 8;
constexpr int kRouterSplitMax = 16;
// The router's partial sums [splits, T, E] get room for kRouterSplitMax splits of
// max(max_tokens, kRouterSplitRows) rows, so that small batches may split K further
// (more CTAs streaming the router weights).
constexpr int kRouterSplitRows = 256;
inline int router_partial_rows(int max_tokens) {
  return kRouterSplitMax * (max_tokens > kRouterSplitRows ? max_tokens : kRouterSplitRows);
}
constexpr int kMaxTpRanks = 8;

// Where the combine writes token t's result: the layer's bf16 output row, or
// (tensor-parallel partial) an fp32 row in the receive slab of the rank that
// owns t: dst[t / rows_per_rank] + (slot * rows_per_rank + t % rows_per_rank) * H.
struct CombineOut {
  __nv_bfloat16* bf16;              // non-null: bf16 [T, H]
  float* dst[kMaxTpRanks];          // otherwise: one slab pointer per owning rank
  int rows_per_rank;
  int slot;
};

// The per-pair return of an expert-parallel rank (signalled sends overlapping
// the down GEMM, [SGLang] MoE 모델을 위한 Single Batch Overlap 기법, §핵심 코드 분석):
// the down GEMM's launch also holds `n_send` CTAs that wait on a per-group
// completion counter (raised by every epilogue warp after it has stored a tile of
// that group) and copy each finished group's expert-output rows, unweighted, into
// the receive slab of the rank that owns the row's token:
//   routed pair (t, j): dst[t / rows] + (j * rows + t % rows) * H
//   shared row of t:    dst[t / rows] + (shared_slot * rows + t % rows) * H
// as fp32 (widened from bf16 on the FP8 path).
struct SendArgs {
  float* dst[kMaxTpRanks];     // one receive slab per owning rank (may be peer memory)
  int rows_per_rank;
  int k;                       // routed slots per row in a slab
  int shared_slot;             // slot of the shared expert's rows (k)
  const int* perm;             // pair index t*k+j of each routed permuted row
  const int* row_token;        // token of each permuted row
  unsigned int* done;          // [G] completion counters, zeroed before the launch
  int n_send;                  // CTAs of the launch that send (0: no sending)
  unsigned int timeout_bit;
};

// ------------------------------------------------------------------ host side

struct GroupedGemmArgs {
  // A (weights): routed experts stacked [E * rows_per_expert, K_routed]; the
  // shared expert [rows_shared, K_shared].  B (activations): [R_cap, K_ld].
  const void* a_routed;
  const void* a_shared;        // may be null when there is no shared group
  const void* b;
  void* d;                     // output rows [R_cap, ldd]: bf16 (gated) or fp32 (down)
  const int* group_offsets;    // [G + 1] on the device
  int E, G;                    // routed experts, total groups (E + S)
  int e_base, n_local;         // a_routed holds experts [e_base, e_base + n_local) only
  int K_routed, K_shared, K_ld;
  int rows_per_expert;         // 2I (gated) or H (down)
  int m_tiles_routed, m_tiles_shared;   // output tiles of 128 weight rows per group
  int up_routed, up_shared;    // gated: row offset of the up half inside a group
  int ldd;
  int R_cap;
  bool gated;
  unsigned int* status;
  unsigned int timeout_bit;
  unsigned long long wait_limit_ns;
  int num_ctas;
  SendArgs send;               // down GEMM only: signalled sends (n_send > 0: cooperative)
};

// e4m3 grouped GEMM with one fp32 scale per 128x128 weight block and per 1x128
// activation group (K blocks of 128).
struct GroupedGemmFp8Args {
  const void* a_routed;        // e4m3 weights [E * rows_per_expert, K_routed]
  const void* a_shared;        // e4m3 weights [rows_shared, K_shared] or null
  const float* sa_routed;      // [E, rows_per_expert / 128, K_routed / 128]
  const float* sa_shared;      // [rows_shared / 128, K_shared / 128]
  const void* b;               // e4m3 activation rows [R_cap, K_ld]
  const float* sb;             // their scales [R_cap, K_ld / 128]
  void* d;                     // gated: e4m3 h [R_cap, ldd]; down: bf16 y [R_cap, ldd]
  float* sd;                   // gated: h scales [R_cap, ldd / 128]
  const int* group_offsets;
  int E, G;
  int e_base, n_local;            // a_routed / sa_routed hold experts [e_base, +n_local) only
  int K_routed, K_shared, K_ld;
  int rows_per_expert;
  int feat_routed, feat_shared;   // output features of a group (gated: I, Is; down: H)
  int up_routed, up_shared;
  int ldd;
  int R_cap;
  bool gated;
  unsigned int* status;
  unsigned int timeout_bit;
  unsigned long long wait_limit_ns;
  int num_ctas;
  SendArgs send;               // down GEMM only: signalled sends (n_send > 0: cooperative)
};

// FP8: quantise every valid token once (1x128 groups) and store codes and scales into
// each of its permuted rows (xp [R, H], sxp [R, H/128]) through the inverse map inv [T, ks].
cudaError_t launch_quant_scatter(const __nv_bfloat16* x, const uint8_t* valid, int T, int H,
                                 const int* inv, int ks, uint8_t* xp, float* sxp, int num_sms,
                                 cudaStream_t st);
cudaError_t launch_grouped_gemm_fp8(const GroupedGemmFp8Args& a, cudaStream_t st);
cudaError_t launch_combine_bf16y(const __nv_bfloat16* y, int H, const int* inv, const float* w,
                                 const uint8_t* valid, int T, int k, int S, const CombineOut& out,
                                 cudaStream_t st);
cudaError_t prepare_grouped_gemm_fp8_kernels();

// Router logits on the tensor cores (router_tc.cu).  W3: [3, E_pad, H] bf16,
// the exact three-part split of Wr (launch_split_router_weights writes it);
// partial: [splits, T, E] fp32.
int router_padded_experts(int E);
cudaError_t launch_split_router_weights(const float* Wr, int E, int H, __nv_bfloat16* W3,
                                        int num_sms, cudaStream_t st);
cudaError_t launch_router_logits_tc(const __nv_bfloat16* x, const uint8_t* valid, int T, int H,
                                    const __nv_bfloat16* W3, int E, float* partial, int splits,
                                    int kb_per_split, unsigned int* status, cudaStream_t st);
cudaError_t prepare_router_kernel();
cudaError_t launch_topk(const float* partial, int splits, const float* bias, const uint8_t* valid,
                        int T, int E, int k, int renorm, float* logits_out, int* ids, float* w,
                        cudaStream_t st);
// scratch: route_scratch_ints(T, E) ints for batches of more than 1024 tokens
// (parallel chunks); nullptr runs the single-block kernel.
int route_scratch_ints(int max_tokens, int E);
cudaError_t launch_route(const int* ids, const uint8_t* valid, int T, int E, int k, int S,
                         int eb, int ee, int* group_offsets, int* perm, int* inv, int* row_token,
                         unsigned int* status, int* scratch, cudaStream_t st);
cudaError_t launch_gather_rows(const __nv_bfloat16* x, int H, const int* row_token,
                               const int* total_rows, int R_cap, __nv_bfloat16* xp,
                               int num_sms, cudaStream_t st);
cudaError_t launch_grouped_gemm(const GroupedGemmArgs& a, cudaStream_t st);
cudaError_t launch_combine(const float* y, int H, const int* inv, const float* w,
                           const uint8_t* valid, int T, int k, int S, const CombineOut& out,
                           cudaStream_t st);
// out[t] = bf16(sum over slots g ascending of slots[g][t]); rows with valid[t] == 0 -> +0.0
cudaError_t launch_reduce_slots(const float* slots, int n_slots, int rows, int H,
                                const uint8_t* valid, __nv_bfloat16* out, cudaStream_t st);
// Owner of a per-pair slab [k + n_extra][rows][H]: out[t] = bf16(sum_j w[t,j] * slab[j][t]
// (fused multiply-adds, j ascending) + sum_s slab[k + s][t] (s ascending)); padding rows +0.0.
cudaError_t launch_reduce_pairs(const float* slab, int k, int n_extra, int rows, int H,
                                const float* w, const uint8_t* valid, __nv_bfloat16* out,
                                cudaStream_t st);
cudaError_t prepare_grouped_gemm_kernels();
const moe_config* plan_config(const moe_plan_s* plan);
void router_split_plan(int T, int E, int H, int num_sms, int partial_rows, int* splits,
                       int* kb_per_split);

// ---------------------------------------------------------------- device side

#if defined(__CUDACC__)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
          bar),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits until the phase with the given parity has completed, for at most
// limit_ns nanoseconds.  On expiry sets `bit` in *status and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  unsigned long long limit_ns,
                                                  unsigned int* status, unsigned int bit) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 >= limit_ns) {
      atomicOr(status, bit);
      return false;
    }
  }
}

// try_wait that lets the hardware suspend the thread for up to hint_ns while
// the phase is incomplete (it resumes when the phase completes), so waiting
// warps do not take issue slots from working ones.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity,
                                                    uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

constexpr uint32_t kSuspendHintNs = 20000;

// Bounded wait with suspension (single thread).
__device__ __forceinline__ bool mbar_wait_sleep(uint32_t bar, uint32_t parity,
                                                unsigned long long limit_ns,
                                                unsigned int* status, unsigned int bit) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, kSuspendHintNs)) return true;
    if (global_timer_ns() - t0 >= limit_ns) {
      atomicOr(status, bit);
      return false;
    }
  }
}

// Bounded wait with suspension taken by a whole warp (warp-uniform result).
__device__ __forceinline__ bool mbar_wait_sleep_warp(uint32_t bar, uint32_t parity,
                                                     unsigned long long limit_ns,
                                                     unsigned int* status, unsigned int bit) {
  if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (__all_sync(0xffffffffu, mbar_try_wait_sleep(bar, parity, kSuspendHintNs))) return true;
    if (__any_sync(0xffffffffu, global_timer_ns() - t0 >= limit_ns)) {
      if ((threadIdx.x & 31) == 0) atomicOr(status, bit);
      return false;
    }
  }
}

// The same wait taken by a whole warp: every lane polls, the warp agrees by
// vote, so a warp never splits between "done" and "expired".
__device__ __forceinline__ bool mbar_wait_bounded_warp(uint32_t bar, uint32_t parity,
                                                       unsigned long long limit_ns,
                                                       unsigned int* status, unsigned int bit) {
  if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    if (__any_sync(0xffffffffu, global_timer_ns() - t0 >= limit_ns)) {
      if ((threadIdx.x & 31) == 0) atomicOr(status, bit);
      return false;
    }
  }
}

// L2 eviction-priority policies for TMA loads.
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 2-D tiled TMA load (no multicast) into this CTA's shared memory; completes
// `bytes` of transaction count on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* m, int x, int y,
                                            uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}

// ---- tcgen05 (5th-generation tensor core, accumulators in tensor memory)

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f8f6f4 (e4m3 inputs, fp32 accumulate), K = 32.
__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor, kind::f8f6f4: fp32 accumulator, e4m3 A and B (format 0),
// both K-major, M = 128, N = n (multiple of 16, 16..256).
__device__ __forceinline__ uint32_t idesc_e4m3_m128(int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// Register reallocation between warpgroups (all four warps of a warpgroup
// execute it).  The shares must add up to the registers the block was
// launched with, or .inc waits forever: launchers check the kernel's register
// count before launching.
template <int N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// L2 eviction priority "normal" (operands reused by other tiles soon).
__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Four 16-column loads of this warp's lanes at four column offsets, one wait.
__device__ __forceinline__ void tmem_ld_16x4(uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             float (&v)[64]) {
  uint32_t r[64];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%16, %17, %18, %19, %20, %21, %22, %23, %24, "
      "%25, %26, %27, %28, %29, %30, %31}, [%65];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%32, %33, %34, %35, %36, %37, %38, %39, %40, "
      "%41, %42, %43, %44, %45, %46, %47}, [%66];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%48, %49, %50, %51, %52, %53, %54, %55, %56, "
      "%57, %58, %59, %60, %61, %62, %63}, [%67];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]),
        "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]),
        "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]),
        "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]),
        "=r"(r[62]), "=r"(r[63])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3)
      : "memory");
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Arrive on an mbarrier once every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// Each thread of the warp reads 32 consecutive 32-bit columns of its own lane.
// The load and its wait are one asm statement, so no use of the registers can
// be scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld_32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Each thread of the warp reads 16 consecutive 32-bit columns of its own lane.
// The load and its wait are one asm statement, so no use of the registers can
// be scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld_16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Each thread of the warp reads 8 consecutive 32-bit columns of its own lane.
// The load and its wait are one asm statement, so no use of the registers can
// be scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld_8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor for a K-major operand tile written by TMA
// with the 128-byte swizzle: rows of 128 bytes, 8-row atoms 1024 bytes apart.
// Fields: start address >> 4 [0,14), leading byte offset >> 4 [16,30) (unused
// for swizzled K-major, set to 1), stride byte offset >> 4 [32,46) = 1024 >> 4,
// version 1 at [46,48), base offset 0, layout type 2 (128B swizzle) at [61,64).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, M = 128, N = n (multiple of 16, 16..256).
__device__ __forceinline__ uint32_t idesc_bf16_m128(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ unsigned int ld_acquire_gpu(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Raised by one lane of an epilogue warp once the warp's stores of a tile of
// group g are done (the warp barrier orders the other lanes' stores before it;
// the fence makes them visible device-wide before the count).
__device__ __forceinline__ void signal_tile_stored(unsigned int* done, int g) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) {
    __threadfence();
    atomicAdd(done + g, 1u);
  }
}

// The send role of a down-GEMM launch with signalled sends: CTA `sid` of `n_send`
// walks the groups in the GEMM's tile order, waits (one thread, bounded) until the
// group's counter reaches `per_tile` x its tile count, then its warps copy their
// share of the group's rows into the owners' slabs.  After an expired wait it
// sets the status bit and stops.  YT: the row type of y (fp32, or bf16 widened).
template <typename YT>
__device__ void send_finished_groups(const SendArgs& sa, const YT* __restrict__ y, int H,
                                     const int* go, const int* ts, int G, int E,
                                     unsigned int per_tile, int sid, unsigned int* status,
                                     unsigned long long limit_ns, int* flag_smem) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int stride = sa.n_send * nwarps;
  for (int g = 0; g < G; ++g) {
    const int beg = go[g], rows = go[g + 1] - beg;
    if (rows == 0) continue;
    if (threadIdx.x == 0) {
      const unsigned int target = per_tile * (unsigned int)(ts[g + 1] - ts[g]);
      int ok = ld_acquire_gpu(sa.done + g) >= target;
      if (!ok) {
        const uint64_t t0 = global_timer_ns();
        while (!(ok = ld_acquire_gpu(sa.done + g) >= target)) {
          if (global_timer_ns() - t0 >= limit_ns) break;
          __nanosleep(256);
        }
      }
      if (!ok) atomicOr(status, sa.timeout_bit);
      *flag_smem = ok;
    }
    __syncthreads();
    const int ok = *flag_smem;
    __syncthreads();
    if (!ok) return;
    for (int i = sid * nwarps + warp; i < rows; i += stride) {
      const int pr = beg + i;
      int t, slot;
      if (g < E) {
        const int pair = sa.perm[pr];
        t = pair / sa.k;
        slot = pair - t * sa.k;
      } else {
        t = sa.row_token[pr];
        slot = sa.shared_slot;
      }
      const int owner = t / sa.rows_per_rank, lt = t - owner * sa.rows_per_rank;
      float* base = sa.dst[0];
#pragma unroll
      for (int r = 1; r < kMaxTpRanks; ++r)
        if (owner == r) base = sa.dst[r];
      float4* dst = reinterpret_cast<float4*>(base + ((size_t)slot * sa.rows_per_rank + lt) * H);
      const YT* src = y + (size_t)pr * H;
      for (int v = lane; v < H / 8; v += 32) {
        float f[8];
        if constexpr (sizeof(YT) == 4) {
          const float4 a = reinterpret_cast<const float4*>(src)[2 * v];
          const float4 b = reinterpret_cast<const float4*>(src)[2 * v + 1];
          f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
          f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
        } else {
          const uint4 r = reinterpret_cast<const uint4*>(src)[v];
          const uint32_t wv[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            f[2 * q] = __uint_as_float(wv[q] << 16);               // bf16 -> fp32, exact
            f[2 * q + 1] = __uint_as_float(wv[q] & 0xffff0000u);
          }
        }
        dst[2 * v] = make_float4(f[0], f[1], f[2], f[3]);
        dst[2 * v + 1] = make_float4(f[4], f[5], f[6], f[7]);
      }
    }
  }
}

#endif  // __CUDACC__

}  // namespace moe
