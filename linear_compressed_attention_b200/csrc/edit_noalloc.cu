// Linear attention step with library-owned scratch (include/edit_attn.h,
// edit_linear_attention_noalloc): for callers that cannot allocate device
// memory. Same kernels as the layer's fp32 path (chunk partials of
// [S_h | z_h], fixed-order combine, apply); only the scratch differs.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "common.cuh"
#include "simt_kernels.cuh"

using namespace edit;

namespace {

// The scratch itself: one per device that loads the library, kept until exit.
static __device__ __align__(256) unsigned char g_noalloc_scratch[EDIT_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device (looked up once).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return EDIT_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return EDIT_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return EDIT_OK;
}

// Plain launch on `st`; the launch's own return code (cudaGetLastError would
// also report, and clear, errors left by the caller's earlier calls).
template <typename... KArgs, typename... Args>
int launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  return cudaLaunchKernelEx(&cfg, kern, args...) == cudaSuccess ? EDIT_OK : EDIT_ERR_CUDA;
}

template <typename T>
int run(const void* q, const void* k, const void* v, int B, int N, int M, int C, int heads, float eps, void* out,
        float* scratch, int chunks, cudaStream_t st) {
  const int d = C / heads;
  const long per_head = static_cast<long>(d) * (d + 1);
  float* part = scratch;                                          // [B][heads][chunks][d][d+1]
  float* Sz = scratch + static_cast<long>(B) * heads * chunks * per_head;  // [B][heads][d][d+1]
  const int nb = (d + 3) / 4;
  int threads = (nb * nb + 31) / 32 * 32;
  if (threads < d) threads = (d + 31) / 32 * 32;
  const size_t smem = 2 * 32 * static_cast<size_t>(d) * sizeof(float);
  int rc = launch(kv_state_partial_kernel<T>, dim3(chunks, heads, B), dim3(threads), smem, st,
                  static_cast<const T*>(k), static_cast<const T*>(v), M, C, heads, chunks, part);
  if (rc != EDIT_OK) return rc;
  const long total = static_cast<long>(B) * heads * per_head;
  const int grid = static_cast<int>((total + 255) / 256 < 4096 ? (total + 255) / 256 : 4096);
  rc = launch(kv_state_combine_kernel, dim3(grid), dim3(256), 0, st, static_cast<const float*>(part), chunks,
              static_cast<int>(per_head), total, Sz);
  if (rc != EDIT_OK) return rc;
  const size_t asmem = static_cast<size_t>(per_head) * sizeof(float);
  if (asmem > 48 * 1024 &&
      cudaFuncSetAttribute(apply_simt_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)asmem) !=
          cudaSuccess)
    return EDIT_ERR_CUDA;
  return launch(apply_simt_kernel<T>, dim3((N + 127) / 128, heads, B), dim3(128), asmem, st,
                static_cast<const T*>(q), static_cast<const float*>(Sz), N, C, heads, eps, static_cast<T*>(out),
                static_cast<float*>(nullptr));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int edit_linear_attention_noalloc(const void* q, const void* k, const void* v, int B, int N, int M,
                                             int C, int heads, int dtype, float attn_eps, void* out,
                                             void* stream) {
  if (!q || !k || !v || !out) return EDIT_ERR_NULL;
  if (dtype != EDIT_F32 && dtype != EDIT_BF16) return EDIT_ERR_DTYPE;
  if (B < 1 || N < 1 || M < 1 || C < 1 || heads < 1 || C % heads != 0) return EDIT_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return EDIT_ERR_ALIGN;
  const int d = C / heads;
  if (d > 128) return EDIT_ERR_UNSUPPORTED;
  if (B > 65535 || heads > 65535) return EDIT_ERR_UNSUPPORTED;  // grid y/z limits
  // blocks of [S | z]: `chunks` partials per (image, head) plus the combined one
  const double block = static_cast<double>(B) * heads * d * (d + 1) * 4.0;
  const double cap = static_cast<double>(EDIT_NOALLOC_SCRATCH_BYTES);
  if (3.0 * block > cap) return EDIT_ERR_SCRATCH;
  int chunks = static_cast<int>(cap / block) - 1;
  const int want = M / 256 > 0 ? M / 256 : 1;
  if (chunks > want) chunks = want;
  if (chunks > 64) chunks = 64;
  if (chunks < 2) chunks = 2;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != EDIT_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* s = static_cast<float*>(scratch);
  return dtype == EDIT_BF16 ? run<__nv_bfloat16>(q, k, v, B, N, M, C, heads, attn_eps, out, s, chunks, st)
                            : run<float>(q, k, v, B, N, M, C, heads, attn_eps, out, s, chunks, st);
}
