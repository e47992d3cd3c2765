// Host-side helpers and the status/introspection entry points of the C ABI.
#include <math.h>
#include <mutex>

#include "host_common.h"

namespace ea {

namespace {

__device__ int g_status_word;

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};
std::mutex g_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

bool encode_tiled(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int rank, const uint64_t* dims,
                  const uint64_t* strides, const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t d[5], s[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) s[i] = strides[i];
  CUresult r = fn(map, dtype, rank, const_cast<void*>(base), d, s, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

int* device_status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  return g_status_ptr[dev];
}

int sm_count_of(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return 0;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sm_count[dev]) {
    // A query about a device that does not exist must not leave an error
    // behind for the next launch's cudaGetLastError check: validate the index
    // first and clear whatever a failed query records.
    int count = 0;
    if (cudaGetDeviceCount(&count) != cudaSuccess || dev >= count) {
      (void)cudaGetLastError();
      return 0;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      (void)cudaGetLastError();
      return 0;
    }
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

int current_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  return sm_count_of(dev);
}

bool encode_bf16_4d(CUtensorMap* map, const void* base, const uint64_t dims[4], const uint64_t strides[3],
                    const uint32_t box[4]) {
  return encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, 4, dims, strides, box);
}

bool encode_u8_4d(CUtensorMap* map, const void* base, const uint64_t dims[4], const uint64_t strides[3],
                  const uint32_t box[4]) {
  return encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, 4, dims, strides, box);
}

bool encode_f32_4d(CUtensorMap* map, const void* base, const uint64_t dims[4], const uint64_t strides[3],
                   const uint32_t box[4]) {
  return encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, base, 4, dims, strides, box);
}

bool encode_bf16_2d(CUtensorMap* map, const void* base, const uint64_t dims[2], const uint64_t strides[1],
                    const uint32_t box[2]) {
  return encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, 2, dims, strides, box);
}

bool encode_bf16_3d(CUtensorMap* map, const void* base, const uint64_t dims[3], const uint64_t strides[2],
                    const uint32_t box[3]) {
  return encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, 3, dims, strides, box);
}

int ensure_smem_attr(const void* kernel, int bytes, int* done_mask) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  // done_mask holds one bit per device (devices >= 32 re-apply every call)
  if (dev < 32 && (__atomic_load_n(done_mask, __ATOMIC_ACQUIRE) & (1 << dev))) return ATTN_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (dev < 32) __atomic_fetch_or(done_mask, 1 << dev, __ATOMIC_RELEASE);
  return ATTN_OK;
}

}  // namespace ea

extern "C" {

int attn_abi_version(void) { return 1; }

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
    case ATTN_ERR_WORKSPACE: return "ATTN_ERR_WORKSPACE";
    default: return "ATTN_ERR_UNKNOWN";
  }
}

int attn_read_device_status(int device) {
  int prev = 0, saved = 0;
  if (cudaGetDevice(&saved) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaSetDevice(device) != cudaSuccess) return ATTN_ERR_CUDA;
  int rc = ATTN_ERR_CUDA;
  int* p = ea::device_status_ptr();
  int zero = 0;
  if (p && cudaDeviceSynchronize() == cudaSuccess &&
      cudaMemcpy(&prev, p, sizeof(int), cudaMemcpyDeviceToHost) == cudaSuccess &&
      cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) == cudaSuccess)
    rc = prev;
  cudaSetDevice(saved);
  return rc;
}

}  // extern "C"
