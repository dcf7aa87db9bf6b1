// Gather-rate probe: how fast can the SMs pull small scattered chunks out of a source buffer into
// shared memory?  It is the ceiling of the sparse attention's gather (every selected 4-token block
// of K and of V is one 2 KB chunk fetched into a shared-memory ring), measured without any of the
// attention's arithmetic.  A source buffer that fits in L2 gives the L2 -> SM ceiling; one much
// larger than L2 gives the HBM gather rate.
//
// Each CTA runs `issuers` warps; warp w owns `stages` stages of `slots` chunk slots and keeps all of
// them in flight: it waits for a stage's previous fill to land, then refills it with chunks from
// pseudo-random chunk-aligned offsets.  Method 0 fills with 1-D bulk copies (cp.async.bulk, the TMA
// engine; one copy per chunk, completion on an mbarrier), method 1 with 16-byte cp.async by all 32
// lanes (the load/store path through L1, bypassed with .cg), method 2 alternates the two by warp.
// Nothing reads the landed data: the probe measures delivery only.  Every wait is bounded.
#include <algorithm>
#include <mutex>

#include "launch.h"
#include "qsa.h"

namespace qsa {
namespace {

struct ProbeArgs {
  const uint8_t* src;
  unsigned long long nchunks;
  int chunk;
  int slots;
  int iters;
  int method;
  unsigned long long seed;
  KernelCtl ctl;
};

__device__ __forceinline__ unsigned long long mix64(unsigned long long x) {
  x ^= x >> 33;
  x *= 0xff51afd7ed558ccdull;
  x ^= x >> 33;
  x *= 0xc4ceb9fe1a85ec53ull;
  x ^= x >> 33;
  return x;
}

__device__ __forceinline__ void cp_async16_cg(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

template <int STAGES>
__global__ void __launch_bounds__(512, 1) gather_probe_kernel(ProbeArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int warps = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t stage_bytes = static_cast<size_t>(a.slots) * a.chunk;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(warps) * STAGES * stage_bytes);
  if (threadIdx.x < warps * STAGES) mbar_init(&bars[threadIdx.x], 1);
  fence_mbar_init();
  __syncthreads();

  uint8_t* ring = smem + static_cast<size_t>(warp) * STAGES * stage_bytes;
  uint64_t* full = bars + warp * STAGES;
  const bool bulk = a.method == 0 || (a.method == 2 && (warp & 1) == 0);
  const unsigned long long stream_id = (static_cast<unsigned long long>(blockIdx.x) * warps + warp) << 32;
  const int pieces = a.chunk / 16;
  int fills = 0;
  bool alive = true;
  for (int it = 0; it < a.iters && alive; ++it) {
    const int st = it % STAGES;
    uint8_t* dst = ring + st * stage_bytes;
    if (bulk) {
      if (it >= STAGES) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(&full[st], ((it / STAGES) - 1) & 1u, a.ctl);
        alive = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      }
      if (!alive) break;
      if (lane == 0) mbar_arrive_expect_tx(&full[st], static_cast<unsigned>(stage_bytes));
      __syncwarp();
      for (int s = lane; s < a.slots; s += 32) {
        const unsigned long long c = mix64(a.seed ^ stream_id ^ (static_cast<unsigned long long>(it) * a.slots + s)) %
                                     a.nchunks;
        bulk_g2s(dst + static_cast<size_t>(s) * a.chunk, a.src + c * a.chunk, a.chunk, &full[st]);
      }
      ++fills;
    } else {
      // keep STAGES - 1 groups in flight while this stage is refilled
      cp_async_wait<STAGES - 1>();
      __syncwarp();
      for (int p = lane; p < a.slots * pieces; p += 32) {
        const int s = p / pieces, off = (p - s * pieces) * 16;
        const unsigned long long c = mix64(a.seed ^ stream_id ^ (static_cast<unsigned long long>(it) * a.slots + s)) %
                                     a.nchunks;
        cp_async16_cg(dst + static_cast<size_t>(s) * a.chunk + off, a.src + c * a.chunk + off);
      }
      cp_async_commit();
    }
  }
  if (bulk) {
    // never leave with a copy in flight: wait for the last fill of every stage
    for (int s = 0; s < STAGES && s < fills; ++s) {
      const int last = s + ((fills - 1 - s) / STAGES) * STAGES;
      mbar_wait(&full[s], (last / STAGES) & 1u, a.ctl);
    }
  } else {
    cp_async_wait<0>();
  }
}

template <int STAGES>
cudaError_t launch_probe(const ProbeArgs& a, int ctas, int issuers, cudaStream_t s) {
  const size_t smem = 128 + static_cast<size_t>(issuers) * STAGES * a.slots * a.chunk + issuers * STAGES * 8;
  cudaError_t e = cudaFuncSetAttribute(gather_probe_kernel<STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  gather_probe_kernel<STAGES><<<ctas, issuers * 32, smem, s>>>(a);
  return cudaPeekAtLastError();
}

}  // namespace
}  // namespace qsa

using namespace qsa;

extern "C" qsa_status_t qsa_probe_gather(const void* src, size_t src_bytes, int chunk_bytes, int method,
                                         int issuer_warps, int stages, int slots_per_warp, int iterations, int ctas,
                                         uint64_t seed, void* stream) {
  if (src == nullptr || (reinterpret_cast<uintptr_t>(src) & 15u) != 0) return QSA_ERR_INVALID_ARGUMENT;
  if (chunk_bytes < 16 || chunk_bytes > 16384 || chunk_bytes % 16 != 0) return QSA_ERR_INVALID_ARGUMENT;
  if (src_bytes < static_cast<size_t>(chunk_bytes)) return QSA_ERR_INVALID_ARGUMENT;
  if (method < 0 || method > 2 || issuer_warps < 1 || issuer_warps > 16 || slots_per_warp < 1 ||
      slots_per_warp > 32 || iterations < 0 || ctas < 0)
    return QSA_ERR_INVALID_ARGUMENT;
  if (stages < 2 || stages > 4) return QSA_ERR_UNSUPPORTED;
  const size_t ring = static_cast<size_t>(issuer_warps) * stages * slots_per_warp * chunk_bytes;
  if (ring + 128 + issuer_warps * stages * 8 > 227u * 1024u) return QSA_ERR_UNSUPPORTED;
  const DeviceInfo* di = device_info();
  if (!di) return QSA_ERR_CUDA;
  if (iterations == 0) return QSA_OK;
  ProbeArgs a{static_cast<const uint8_t*>(src), src_bytes / chunk_bytes, chunk_bytes, slots_per_warp, iterations,
              method, seed, kernel_ctl(di)};
  const int grid = ctas ? ctas : di->num_sms;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = stages == 2 ? launch_probe<2>(a, grid, issuer_warps, s)
                  : stages == 3 ? launch_probe<3>(a, grid, issuer_warps, s)
                                : launch_probe<4>(a, grid, issuer_warps, s);
  return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}
