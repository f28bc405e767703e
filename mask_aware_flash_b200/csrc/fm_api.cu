// Host-side plumbing shared by the entry points: status strings, the
// per-device status word, and TMA tensor-map encoding.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "fm_common.cuh"

namespace fm {

// Latched device-side error (FM_ERR_DEVICE_TIMEOUT << 16 | site), one per device, and the slot into
// which fm_get_device_status moves it (read and cleared in one atomic exchange).
__device__ int g_fm_status;
__device__ int g_fm_status_taken;

namespace {
std::mutex g_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

EncodeTiledFn get_encode() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  return g_encode;
}
}  // namespace

// Device address of the status word on the current device, looked up on every call (a cached
// address would go stale after cudaDeviceReset or a new primary context).
int* device_status_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_fm_status) != cudaSuccess) return nullptr;
  return static_cast<int*>(p);
}

// 4-D map over a [B, n, H, D] bf16 tensor: dims (D, H, n, B), box (64, 1, box_rows, 1),
// 128-byte swizzle (one 64-element row of the box = one swizzle span).
bool encode_tmap_bf16_4d(CUtensorMap* map, const void* base, uint64_t D, uint64_t H, uint64_t n, uint64_t B,
                         uint32_t box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[4] = {D, H, n, B};
  cuuint64_t strides[3] = {D * 2, H * D * 2, n * H * D * 2};
  cuuint32_t box[4] = {64, 1, box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Same view of a [B, n, H, D] fp32 tensor: box (32, 1, box_rows, 1), 32 fp32 = one swizzle span.
bool encode_tmap_f32_4d(CUtensorMap* map, const void* base, uint64_t D, uint64_t H, uint64_t n, uint64_t B,
                        uint32_t box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[4] = {D, H, n, B};
  cuuint64_t strides[3] = {D * 4, H * D * 4, n * H * D * 4};
  cuuint32_t box[4] = {32, 1, box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// One CTA waits on an mbarrier that nothing arrives on.  The bounded wait gives
// up after kTimeoutNs and records FM_ERR_DEVICE_TIMEOUT (site 0x7E57) in the
// device status word; the kernel then returns normally.
__global__ void selftest_wait_kernel(int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(smem_u32(&bar), 0, &abort_flag)) record_failure(status, &abort_flag, 0x7E57);
}


// Moves the status word into `taken` and clears it in one atomic exchange, so a failure that a
// kernel on another stream latches concurrently is either returned now or kept for the next read.
__global__ void take_status_kernel(int* status, int* taken) { *taken = atomicExch(status, 0); }

}  // namespace fm

extern "C" {

fm_status fm_selftest_wait_timeout(fm_stream_t stream) {
  int* st = fm::device_status_ptr();
  if (!st) return FM_ERR_CUDA;
  fm::selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(st);
  return cudaGetLastError() == cudaSuccess ? FM_OK : FM_ERR_CUDA;
}

const char* fm_status_string(fm_status s) {
  switch (s) {
    case FM_OK: return "ok";
    case FM_ERR_INVALID_ARG: return "invalid argument";
    case FM_ERR_UNSUPPORTED: return "unsupported problem shape or type";
    case FM_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case FM_ERR_CUDA: return "CUDA call or kernel launch failed";
    case FM_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait ran out on the device";
    case FM_ERR_DEVICE_CHECK: return "a device-side index or canary check failed (debug build)";
  }
  return "unknown status";
}

fm_status fm_get_device_status(fm_stream_t stream) {
  int* p = fm::device_status_ptr();
  void* taken = nullptr;
  if (!p || cudaGetSymbolAddress(&taken, fm::g_fm_status_taken) != cudaSuccess) return FM_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  fm::take_status_kernel<<<1, 1, 0, s>>>(p, static_cast<int*>(taken));
  int v = 0;
  if (cudaGetLastError() != cudaSuccess || cudaMemcpyAsync(&v, taken, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return FM_ERR_CUDA;
  return v == 0 ? FM_OK : static_cast<fm_status>(v >> 16);
}

}  // extern "C"
