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

// Methods 3 and 4: tiled tensor copies (cp.async.bulk.tensor, 128-byte swizzle) of one 4-token block
// from a 3-D map over the source viewed as [tokens][2 heads][128 d] bf16: method 3 copies boxes of
// [4 tokens][1 head][64 d] (512 bytes, four per block and tensor, as the query-tile attention does),
// method 4 boxes of [4 tokens][2 heads][64 d] (1 KB).  `slots` boxes per stage and warp.
template <int STAGES>
__global__ void __launch_bounds__(512, 1) tensor_probe_kernel(const __grid_constant__ CUtensorMap map, ProbeArgs a,
                                                              int box_bytes) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warps = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t stage_bytes = static_cast<size_t>(a.slots) * box_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(warps) * STAGES * stage_bytes);
  if (threadIdx.x < warps * STAGES) mbar_init(&bars[threadIdx.x], 1);
  fence_mbar_init();
  __syncthreads();
  uint8_t* ring = smem + static_cast<size_t>(warp) * STAGES * stage_bytes;
  uint64_t* full = bars + warp * STAGES;
  const unsigned long long stream_id = (static_cast<unsigned long long>(blockIdx.x) * warps + warp) << 32;
  const unsigned long long nblocks = a.nchunks;   // 4-token blocks in the source
  int fills = 0;
  bool alive = true;
  for (int it = 0; it < a.iters && alive; ++it) {
    const int st = it % STAGES;
    uint8_t* dst = ring + st * stage_bytes;
    if (it >= STAGES) {
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&full[st], ((it / STAGES) - 1) & 1u, a.ctl);
      alive = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    if (!alive) break;
    if (lane == 0) mbar_arrive_expect_tx(&full[st], static_cast<unsigned>(stage_bytes));
    __syncwarp();
    for (int sl = lane; sl < a.slots; sl += 32) {
      const unsigned long long r = mix64(a.seed ^ stream_id ^ (static_cast<unsigned long long>(it) * a.slots + sl));
      const int blk = static_cast<int>(r % nblocks);
      const int half = static_cast<int>((r >> 40) & 1), head = static_cast<int>((r >> 41) & 1);
      tma_load_3d(dst + static_cast<size_t>(sl) * box_bytes, &map, &full[st], half * 64, box_bytes == 512 ? head : 0,
                  blk * 4);
    }
    ++fills;
  }
  for (int sidx = 0; sidx < STAGES && sidx < fills; ++sidx) {
    const int last = sidx + ((fills - 1 - sidx) / STAGES) * STAGES;
    mbar_wait(&full[sidx], (last / STAGES) & 1u, a.ctl);
  }
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

template <int STAGES>
cudaError_t launch_tensor_probe(const ProbeArgs& a, int ctas, int issuers, int box_bytes, cudaStream_t s) {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  if (!fn) return cudaErrorInvalidValue;
  CUtensorMap map;
  const unsigned long long tokens = a.nchunks * 4;
  cuuint64_t dims[3] = {128, 2, tokens};
  cuuint64_t strides[2] = {256, 512};
  cuuint32_t box[3] = {64, box_bytes == 512 ? 1u : 2u, 4};
  cuuint32_t estr[3] = {1, 1, 1};
  if (fn(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint8_t*>(a.src), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + static_cast<size_t>(issuers) * STAGES * a.slots * box_bytes + issuers * STAGES * 8;
  cudaError_t e = cudaFuncSetAttribute(tensor_probe_kernel<STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  tensor_probe_kernel<STAGES><<<ctas, issuers * 32, smem, s>>>(map, a, box_bytes);
  return cudaPeekAtLastError();
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
  QSA_NVTX();
  if (src == nullptr || (reinterpret_cast<uintptr_t>(src) & 15u) != 0) return QSA_ERR_INVALID_ARGUMENT;
  if (chunk_bytes < 16 || chunk_bytes > 16384 || chunk_bytes % 16 != 0) return QSA_ERR_INVALID_ARGUMENT;
  if (src_bytes < static_cast<size_t>(chunk_bytes)) return QSA_ERR_INVALID_ARGUMENT;
  if (method < 0 || method > 4 || issuer_warps < 1 || issuer_warps > 16 || slots_per_warp < 1 ||
      slots_per_warp > 32 || iterations < 0 || ctas < 0)
    return QSA_ERR_INVALID_ARGUMENT;
  // tensor boxes: 512 bytes (method 3) or 1 KB (method 4) from a source of whole 2 KB blocks
  if (method >= 3 && (chunk_bytes != (method == 3 ? 512 : 1024) || src_bytes < 2048)) return QSA_ERR_INVALID_ARGUMENT;
  if (stages < 2 || stages > 4) return QSA_ERR_UNSUPPORTED;
  const size_t ring = static_cast<size_t>(issuer_warps) * stages * slots_per_warp * chunk_bytes;
  if (ring + 1024 + issuer_warps * stages * 8 > 227u * 1024u) return QSA_ERR_UNSUPPORTED;
  const DeviceInfo* di = device_info();
  if (!di) return QSA_ERR_CUDA;
  if (iterations == 0) return QSA_OK;
  ProbeArgs a{static_cast<const uint8_t*>(src), src_bytes / chunk_bytes, chunk_bytes, slots_per_warp, iterations,
              method, seed, kernel_ctl(di)};
  const int grid = ctas ? ctas : di->num_sms;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (method >= 3) {
    a.nchunks = src_bytes / 2048;   // whole 4-token blocks of [4][2][128] bf16
    cudaError_t e = stages == 2 ? launch_tensor_probe<2>(a, grid, issuer_warps, chunk_bytes, s)
                    : stages == 3 ? launch_tensor_probe<3>(a, grid, issuer_warps, chunk_bytes, s)
                                  : launch_tensor_probe<4>(a, grid, issuer_warps, chunk_bytes, s);
    return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
  }
  cudaError_t e = stages == 2 ? launch_probe<2>(a, grid, issuer_warps, s)
                  : stages == 3 ? launch_probe<3>(a, grid, issuer_warps, s)
                                : launch_probe<4>(a, grid, issuer_warps, s);
  return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}
