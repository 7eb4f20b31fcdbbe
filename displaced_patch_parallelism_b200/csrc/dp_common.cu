// dp_common.cu -- error reporting, the device status word, TMA descriptor
// encoding and the small ABI helpers.
#include <cudaTypedefs.h>
#include <stdarg.h>
#include <stdio.h>

#include <mutex>

#include <cstdlib>

#include "dp_common.cuh"

namespace dp {

// One status word per device that loads the library: kernels record a
// bounded wait that ran out here (DP_ERR_TIMEOUT); dp_device_status reads
// and clears it.
__device__ int g_status_word = 0;

static thread_local char t_last_error[512] = "";
// The status word of the block step running on this thread (null: none).
static thread_local int* t_status_word = nullptr;

StatusScope::StatusScope(int* word) : prev_(t_status_word) { t_status_word = word; }
StatusScope::~StatusScope() { t_status_word = prev_; }

struct LaunchRecorder {
  void* const* events = nullptr;
  int n = 0;
  int idx = 0;
};
static thread_local LaunchRecorder t_rec;

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = getenv("DP_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

void mark_launch(cudaStream_t s) {
  if (t_rec.events && t_rec.idx < t_rec.n)
    cudaEventRecord(static_cast<cudaEvent_t>(t_rec.events[t_rec.idx++]), s);
}

void recorder_begin(void* const* events, int n) {
  t_rec.events = events;
  t_rec.n = n;
  t_rec.idx = 0;
}

int recorder_end() {
  const int used = t_rec.idx;
  t_rec.events = nullptr;
  t_rec.n = 0;
  t_rec.idx = 0;
  return used;
}

int set_error(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return DP_OK;
  return set_error(DP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int* device_status_ptr() {
  if (t_status_word) return t_status_word;
  static int* ptrs[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int*>(p);
  }
  return ptrs[dev];
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

int encode_tmap(CUtensorMap* map, CUtensorMapDataType dt, int rank, void* base,
                const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                CUtensorMapSwizzle swizzle) {
  auto fn = get_encode_fn();
  if (!fn) return set_error(DP_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, dt, rank, base, dims, strides_bytes, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return set_error(DP_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d), rank %d", (int)r, rank);
  return DP_OK;
}

int read_clear_status(int* word, cudaStream_t s, int* out) {
  int host = 0;
  int rc = cuda_check(cudaMemcpyAsync(&host, word, sizeof(int), cudaMemcpyDeviceToHost, s),
                      "read status");
  if (rc) return rc;
  rc = cuda_check(cudaStreamSynchronize(s), "sync for status");
  if (rc) return rc;
  if (host != 0) {
    rc = cuda_check(cudaMemsetAsync(word, 0, sizeof(int), s), "clear status");
    if (rc) return rc;
    rc = cuda_check(cudaStreamSynchronize(s), "sync after clear");
    if (rc) return rc;
  }
  *out = host;
  return DP_OK;
}

}  // namespace dp

extern "C" {

const char* dp_last_error(void) { return dp::t_last_error; }

const char* dp_version(void) { return "dp-b200 0.1 (sm_100a)"; }

int dp_mode_for_step(int step, int warmup) {
  if (step < 0 || warmup < 0) return dp::set_error(DP_ERR_INVALID_ARG, "negative step/warmup");
  if (step < warmup) return DP_MODE_SYNC;
  if (step == 0) return DP_MODE_NAIVE;
  return DP_MODE_DISPLACED;
}

int dp_device_status(void* stream, int* status) {
  if (!status) return dp::set_error(DP_ERR_INVALID_ARG, "status is NULL");
  int* p = dp::device_status_ptr();
  if (!p) return dp::set_error(DP_ERR_CUDA, "status word address unavailable");
  return dp::read_clear_status(p, static_cast<cudaStream_t>(stream), status);
}

}  // extern "C"
