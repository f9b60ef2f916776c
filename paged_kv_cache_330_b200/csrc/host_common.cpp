// Status strings, the device error word aggregate, and the tensor-map encoder
// (the driver entry point is fetched through the runtime, so the library does
// not link libcuda directly).

#include "host_common.h"

#include <atomic>
#include <mutex>

extern "C" int pa__err_write_kv(unsigned int* out);
extern "C" int pa__err_decode(unsigned int* out);
extern "C" int pa__err_prefill(unsigned int* out);
extern "C" int pa__err_rope(unsigned int* out);
extern "C" int pa__err_int8(unsigned int* out);

extern "C" const char* pa_strerror(int status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID: return "PA_ERR_INVALID: invalid argument";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED: unsupported shape or dtype";
    case PA_ERR_ALIGN: return "PA_ERR_ALIGN: pointer not 16-byte aligned";
    case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE: workspace missing or too small";
    case PA_ERR_CUDA: return "PA_ERR_CUDA: CUDA call failed";
    case PA_ERR_OOM: return "PA_ERR_OOM: not enough free blocks";
    case PA_ERR_NOT_FOUND: return "PA_ERR_NOT_FOUND: unknown or duplicate sequence id";
    case PA_ERR_DEVICE: return "PA_ERR_DEVICE: a kernel recorded a device-side error";
    default: return "unknown status";
  }
}

extern "C" const char* pa_version(void) { return "0.1.0"; }

extern "C" int pa_copy_async(void* dst, const void* src, size_t bytes, void* stream) {
  if (bytes == 0) return PA_OK;
  if (!dst || !src) return PA_ERR_INVALID;
  return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDefault, (cudaStream_t)stream) == cudaSuccess ? PA_OK
                                                                                               : PA_ERR_CUDA;
}

extern "C" int pa_device_error(int* out) {
  if (!out) return PA_ERR_INVALID;
  if (cudaDeviceSynchronize() != cudaSuccess) return PA_ERR_CUDA;
  unsigned int a = 0, b = 0, c = 0, d = 0, e = 0;
  int s;
  if ((s = pa__err_write_kv(&a)) != PA_OK) return s;
  if ((s = pa__err_decode(&b)) != PA_OK) return s;
  if ((s = pa__err_prefill(&c)) != PA_OK) return s;
  if ((s = pa__err_rope(&d)) != PA_OK) return s;
  if ((s = pa__err_int8(&e)) != PA_OK) return s;
  *out = (int)(a | b | c | d | e);
  return PA_OK;
}

namespace pa {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  try {
    std::call_once(once, [] {
      void* p = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
          q == cudaDriverEntryPointSuccess)
        fn = reinterpret_cast<EncodeTiledFn>(p);
    });
  } catch (...) {  // no exception leaves the C ABI; the caller reports PA_ERR_CUDA
    return nullptr;
  }
  return fn;
}

int encode_2d_sw128(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t row_stride_bytes,
                    uint32_t box_cols, uint32_t box_rows) {
  return encode_2d_u16(map, base, cols, rows, row_stride_bytes, box_cols, box_rows, 128);
}

int encode_2d_u16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t row_stride_bytes,
                  uint32_t box_cols, uint32_t box_rows, uint32_t swizzle_bytes, uint32_t l2_fill_bytes) {
  if (swizzle_bytes != 128 && swizzle_bytes != 64) return PA_ERR_CUDA;
  EncodeTiledFn fn = get_encode();
  if (!fn) return PA_ERR_CUDA;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                  l2_fill_bytes == 128 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B : CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PA_OK : PA_ERR_CUDA;
}

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  static std::atomic<int> cache[64];  // zero-initialised; calls from several host threads may race to fill it
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

}  // namespace pa
