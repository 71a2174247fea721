// moe_route_from_logits_noalloc: routing from given logits for callers that
// cannot allocate device memory (see include/moe.h).  The scratch that
// moe_route_from_logits takes from the caller's workspace lives here, in one
// file-scope device array.  The results are identical to that call's: the same
// top-k kernel, and the routing kernel that moe_route_from_logits runs up to
// 1024 tokens (above that the workspace path splits the counting over parallel
// kernels with the same deterministic result; here one block walks the chunks).
#include <mutex>

#include "moe_internal.cuh"

#define MOE_EXPORT extern "C" __attribute__((visibility("default")))

namespace {

// Loaded with the library on every GPU that uses it, freed at process exit.
static __device__ __align__(256) unsigned char g_route_scratch[MOE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
// Device address of g_route_scratch per device, looked up once.  In host code
// the symbol names a host-side shadow, never the device memory itself.
void* g_scratch_dev[kMaxDevices] = {};
std::mutex g_scratch_mutex;

size_t round256(size_t n) { return (n + 255) / 256 * 256; }

moe_status scratch_for_current_device(unsigned char** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return MOE_ERR_CUDA;
  if (dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_dev[dev] == nullptr) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (major != 10 || minor != 0) return MOE_ERR_UNSUPPORTED;   // built for sm_100a only
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr)
      return MOE_ERR_CUDA;
    g_scratch_dev[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_scratch_dev[dev]);
  return MOE_OK;
}

}  // namespace

MOE_EXPORT moe_status moe_route_from_logits_noalloc(moe_plan_t plan, const float* logits,
                                                    const uint8_t* valid, int T, int k,
                                                    int* topk_ids, float* topk_w, int* perm,
                                                    int* offsets, void* stream) {
  if (plan == nullptr) return MOE_ERR_INVALID_ARG;
  const moe_config& c = *moe::plan_config(plan);
  if (T < 0 || T > c.max_tokens || k < 1 || k > c.top_k_max) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (logits == nullptr || topk_ids == nullptr || topk_w == nullptr || perm == nullptr ||
      offsets == nullptr)
    return MOE_ERR_INVALID_ARG;
  const size_t E = (size_t)c.num_experts, S = (size_t)c.num_shared;
  const size_t ks = (size_t)k + S;
  // layout: status | group offsets | inverse | row -> token (the logits are not copied)
  const size_t off_goff = 256;
  const size_t off_inv = off_goff + round256(sizeof(int) * (E + 2));
  const size_t off_rowtok = off_inv + round256(sizeof(int) * (size_t)T * ks);
  const size_t need = off_rowtok + round256(sizeof(int) * (size_t)T * ks);
  if (need > MOE_STATIC_SCRATCH_BYTES) return MOE_ERR_UNSUPPORTED;

  unsigned char* scratch = nullptr;
  moe_status s = scratch_for_current_device(&scratch);
  if (s != MOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned int* status = reinterpret_cast<unsigned int*>(scratch);
  int* goff = reinterpret_cast<int*>(scratch + off_goff);
  if (cudaMemsetAsync(status, 0, sizeof(unsigned int), st) != cudaSuccess) return MOE_ERR_CUDA;
  if (moe::launch_topk(logits, 1, nullptr, valid, T, (int)E, k, c.renormalize, nullptr,
                       topk_ids, topk_w, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (moe::launch_route(topk_ids, valid, T, (int)E, k, (int)S, 0, (int)E, goff, perm,
                        reinterpret_cast<int*>(scratch + off_inv),
                        reinterpret_cast<int*>(scratch + off_rowtok), status, nullptr,
                        st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaMemcpyAsync(offsets, goff, sizeof(int) * (E + 1), cudaMemcpyDeviceToDevice, st) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
