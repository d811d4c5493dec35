// lt_abi.cu -- status strings, ABI version and shared host helpers.
#include <mutex>

#include "lt_common.cuh"

namespace lt {

int num_sms() {
  // cached per device; B200 has 148
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

int blocks_per_sm(const void *kernel, int threads, size_t dyn_smem) {
  struct Entry {
    const void *k;
    int dev, threads;
    size_t smem;
    int blocks;
  };
  static Entry cache[128];
  static int used = 0;
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].k == kernel && cache[i].dev == dev && cache[i].threads == threads && cache[i].smem == dyn_smem)
      return cache[i].blocks;
  int b = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kernel, threads, dyn_smem) != cudaSuccess || b < 1) {
    cudaGetLastError();
    b = 1;
  }
  if (used < 128) cache[used++] = Entry{kernel, dev, threads, dyn_smem, b};
  return b;
}

lt_status launch_status() { return cudaGetLastError() == cudaSuccess ? LT_OK : LT_ERR_CUDA; }

void *driver_fn(const char *name) {
  // the CUDA driver API through the runtime's entry-point lookup, so that the
  // library does not link libcuda itself (it loads on hosts without a GPU)
  void *fn = nullptr;
  cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
  if (cudaGetDriverEntryPointByVersion(name, &fn, 12000, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return fn;
}

bool current_context_id(unsigned long long *id) {
  typedef int (*ctx_get_current_t)(void **);
  typedef int (*ctx_get_id_t)(void *, unsigned long long *);
  static ctx_get_current_t get_current = nullptr;
  static ctx_get_id_t get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    get_current = (ctx_get_current_t)driver_fn("cuCtxGetCurrent");
    get_id = (ctx_get_id_t)driver_fn("cuCtxGetId");
  });
  void *ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != 0 || !ctx) return false;
  return get_id(ctx, id) == 0;
}

}  // namespace lt

LT_API const char *lt_status_string(lt_status s) {
  switch (s) {
    case LT_OK:
      return "ok";
    case LT_ERR_INVALID_ARG:
      return "invalid argument";
    case LT_ERR_MISALIGNED:
      return "misaligned pointer";
    case LT_ERR_UNSUPPORTED:
      return "unsupported parameters";
    case LT_ERR_CORRUPT_STREAM:
      return "corrupt compressed stream";
    case LT_ERR_SIZE_MISMATCH:
      return "decoded size differs from the declared size";
    case LT_ERR_CUDA:
      return "CUDA launch failed";
    case LT_ERR_TIMEOUT:
      return "an on-chip wait ran out (internal error)";
    case LT_ERR_CHECKSUM:
      return "block checksum mismatch";
  }
  return "unknown status";
}

LT_API int32_t lt_abi_version(void) { return LT_ABI_VERSION; }
