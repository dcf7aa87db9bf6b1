// qsa_sparse_attn_decode_noalloc: split-KV decode whose partial results live in a scratch array
// compiled into the library, for callers that cannot allocate device memory (see qsa.h).
#include <algorithm>
#include <mutex>

#include "launch.h"
#include "qsa.h"

namespace qsa {
namespace {

// One array per GPU that loads the library; shared by every call on that GPU.
static __device__ __align__(256) float g_decode_scratch[QSA_NOALLOC_DECODE_SCRATCH_BYTES / sizeof(float)];

constexpr int kMaxDevices = 64;
std::once_flag g_once[kMaxDevices];
float* g_scratch_ptr[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];

// Device address of the array on the current device.  In host code the array's name is only a
// host-side handle, so the address must be looked up once per device, with that device current.
float* scratch_for(int dev, cudaError_t* err) {
  std::call_once(g_once[dev], [dev] {
    void* p = nullptr;
    g_scratch_err[dev] = cudaGetSymbolAddress(&p, g_decode_scratch);
    g_scratch_ptr[dev] = g_scratch_err[dev] == cudaSuccess ? static_cast<float*>(p) : nullptr;
  });
  *err = g_scratch_err[dev];
  return g_scratch_ptr[dev];
}

bool ok_ptr(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace qsa

using namespace qsa;

extern "C" qsa_status_t qsa_sparse_attn_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                                                       const int32_t* seqlens, const int32_t* idx, int B, int Lmax,
                                                       int Hq, int Hkv, int D, int k_blocks, int blk, float scale,
                                                       int num_splits, void* out, float* lse, void* stream) {
  QSA_NVTX();
  if (Hq < 1 || Hkv < 1 || k_blocks < 0 || Hq % Hkv) return QSA_ERR_INVALID_ARGUMENT;
  if ((D != 128 && D != 256) || blk != 4 || Hkv > 2 || Hq / Hkv > 16) return QSA_ERR_UNSUPPORTED;
  if (B < 0 || Lmax < 1 || num_splits < 0) return QSA_ERR_INVALID_ARGUMENT;
  if (B == 0) return QSA_OK;
  if (!ok_ptr(q) || !ok_ptr(kcache) || !ok_ptr(vcache) || !ok_ptr(out) || seqlens == nullptr ||
      (k_blocks > 0 && idx == nullptr))
    return QSA_ERR_INVALID_ARGUMENT;
  const size_t per_split = static_cast<size_t>(B) * Hq * (D + 2) * sizeof(float);
  const int fit = static_cast<int>(std::min<size_t>(QSA_NOALLOC_DECODE_SCRATCH_BYTES / per_split, 1 << 20));
  const DeviceInfo* di = device_info();
  if (!di) return QSA_ERR_CUDA;
  // The split count the launch really uses (never more splits than listed blocks) is what must fit.
  int splits = num_splits == 0 ? std::min(decode_default_splits(di, B, std::max(k_blocks, 1)), std::max(fit, 1))
                               : num_splits;
  splits = std::max(1, std::min(splits, std::max(k_blocks, 1)));
  if (splits > 1 && splits > fit) return QSA_ERR_WORKSPACE_TOO_SMALL;
  float* part = nullptr;
  if (splits > 1) {
    cudaError_t e;
    part = scratch_for(di->device, &e);
    if (e != cudaSuccess || part == nullptr) return QSA_ERR_CUDA;
  }
  cudaError_t e = launch_attn_decode(di, q, kcache, vcache, seqlens, idx, B, Lmax, Hq, Hkv, D, k_blocks, scale, splits,
                                     out, lse, part, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}
