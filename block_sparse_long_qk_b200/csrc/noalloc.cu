// fp_pool_and_mask_noalloc: pooling and mask building without any device allocation.
//
// The regular path needs the pooled means q_pool / k_pool as intermediate buffers between the
// pool kernel and the mask kernel, and the caller allocates them. Some callers cannot allocate
// device memory at that point: a serving engine that hands nearly all free HBM to its KV-cache
// pool at start-up and runs requests on a fixed memory budget, code whose calls must not
// synchronize the device (cudaMalloc and cudaFree do), or a host application that passes the
// library only its preallocated input and output buffers. For them this entry keeps the
// pooled means in a file-scope device array of fixed size instead.
//
// The array is part of the library image: every GPU that loads the library holds its
// kNoAllocPoolFloats floats (32 MiB) until the process exits. All calls share it; each call
// overwrites every pooled value it later reads, so nothing needs clearing between calls, but
// two calls whose work overlaps on the same GPU (for instance on two streams) race on the
// array. Each GPU has its own copy, so calls on different GPUs do not interfere.
//
// The array's device address is looked up once per device and kept for the life of the
// process, so the entry must not be used on a device after cudaDeviceReset (which destroys the
// context the address belongs to).
//
// The mask here always converts the pooled keys to the bf16 hi / lo tensor-core operands inside
// the mask kernel (no k_pool_split buffer exists to load them from), and no workspace is taken:
// the kernels still refuse inconsistent prefix sums and bound every wait, but a failure is not
// reported through a status word.
#include <mutex>

#include "fp_common.cuh"
#include "fp_launch.h"

namespace {

// Capacity of the pooled scratch: (Hq + Hkv) * total_blocks * d floats at most.
// 8 Mi floats = 32 MiB covers e.g. Hq = 32, Hkv = 8, d = 128 up to 1638 blocks (209K tokens at
// block 128).
constexpr size_t kNoAllocPoolFloats = size_t(8) << 20;

static __device__ __align__(256) float g_pool_scratch[kNoAllocPoolFloats];

constexpr int kMaxDevices = 64;
float* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_pool_scratch on the current device, looked up once per device. In host
// code the symbol itself is only a host-side stand-in, never a device address.
cudaError_t scratch_address(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_pool_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int fp_pool_and_mask_noalloc(
    const void* q, const void* k, int dtype, const float* q_scale, const float* k_scale,
    const int32_t* cu_seqlens, const int32_t* cu_blocks, int batch, int total_tokens,
    int total_blocks, int max_blocks, int Hq, int Hkv, int d, int block,
    const int32_t* k_page_table, int page_size, int max_pages, int num_pages, float alpha,
    float scale, int flags, uint32_t* mask_bits, int32_t* kv_cnt, int32_t* kv_idx,
    void* stream) {
  if (Hq <= 0 || Hkv <= 0 || d <= 0 || total_blocks < 0)
    return fp::set_error(FP_ERR_INVALID_ARG, "bad head count, head dim or block count");
  const size_t need = (static_cast<size_t>(Hq) + Hkv) * static_cast<size_t>(total_blocks) * d;
  if (need > kNoAllocPoolFloats)
    return fp::set_error(FP_ERR_INVALID_ARG,
                         "fp_pool_and_mask_noalloc: the pooled means need %zu floats "
                         "((Hq + Hkv) * total_blocks * d) but the static scratch holds %zu "
                         "(32 MiB); use fp_pool_qk + fp_build_block_mask with caller buffers",
                         need, kNoAllocPoolFloats);
  float* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess)
    return fp::set_error(FP_ERR_CUDA, "cudaGetSymbolAddress of the pooled scratch: %s",
                         cudaGetErrorString(e));
  float* q_pool = scratch;
  float* k_pool = scratch + static_cast<size_t>(Hq) * total_blocks * d;
  int rc = fp_pool_qk(q, k, dtype, q_scale, k_scale, cu_seqlens, cu_blocks, batch, total_tokens,
                      total_blocks, Hq, Hkv, d, block, k_page_table, page_size, max_pages,
                      num_pages, q_pool, k_pool, nullptr, nullptr, stream);
  if (rc != FP_OK) return rc;
  return fp_build_block_mask(q_pool, k_pool, nullptr, cu_blocks, batch, total_blocks, max_blocks,
                             Hq, Hkv, d, alpha, scale, flags, mask_bits, kv_cnt, kv_idx, nullptr,
                             stream);
}
