// api_common.cu -- libdsq entry points that launch nothing (sizes, status,
// errors, version) and the host plumbing declared in dsq_host.h.
#include <atomic>
#include <cstdarg>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "../../include/dsq_test.h"
#include "dsq_host.h"

namespace dsq {

// Device status word, one per device (each device has its own copy of a
// __device__ variable).  Kernels receive its address as an argument.
static __device__ uint32_t g_status_word;

namespace {
thread_local char t_error[512] = "no error";
std::atomic<uint64_t> g_launches{0};
std::atomic<uint64_t> g_wait_limit_ns{1000ull * 1000ull * 1000ull};

std::mutex g_dev_mu;
struct DevState {
  uint64_t ctx = 0;   // context the entries below belong to (0: none yet)
  int ok = DSQ_ERR_UNSUPPORTED_DEVICE;
  uint32_t *status = nullptr;
  int sms = 0;
};
DevState g_dev[kMaxDevices];

PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;
std::once_flag g_ctx_fns_once;

void load_ctx_fns() {
  void *p = nullptr;
  cudaDriverEntryPointQueryResult q{};
  if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  p = nullptr;
  if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
}
}  // namespace

int current_context(int *device, uint64_t *ctx_id) {
  cudaError_t e = cudaGetDevice(device);
  if (e != cudaSuccess) return fail(DSQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (*device < 0 || *device >= kMaxDevices) return fail(DSQ_ERR_UNSUPPORTED_DEVICE, "device %d", *device);
  std::call_once(g_ctx_fns_once, load_ctx_fns);
  if (g_ctx_current == nullptr || g_ctx_id == nullptr)
    return fail(DSQ_ERR_CUDA, "cuCtxGetCurrent / cuCtxGetId are not available from the driver");
  for (int attempt = 0; attempt < 2; ++attempt) {
    CUcontext c = nullptr;
    if (g_ctx_current(&c) != CUDA_SUCCESS) return fail(DSQ_ERR_CUDA, "cuCtxGetCurrent failed");
    if (c != nullptr) {
      unsigned long long id = 0;
      if (g_ctx_id(c, &id) != CUDA_SUCCESS) return fail(DSQ_ERR_CUDA, "cuCtxGetId failed");
      *ctx_id = static_cast<uint64_t>(id) + 1;   // never 0
      return DSQ_OK;
    }
    // No context is current on this thread yet: the runtime binds the
    // device's primary context on its first call that needs one.
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_status_word);
    if (e != cudaSuccess) return fail(DSQ_ERR_CUDA, "cudaGetSymbolAddress(status): %s", cudaGetErrorString(e));
  }
  return fail(DSQ_ERR_CUDA, "no CUDA context is current");
}

int fail(int code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_error, sizeof(t_error), fmt, ap);
  va_end(ap);
  return code;
}

int device_ready(uint32_t **status_word, int *num_sms) {
  int dev = -1;
  uint64_t ctx = 0;
  int rc = current_context(&dev, &ctx);
  if (rc != DSQ_OK) return rc;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevState &s = g_dev[dev];
  if (s.ctx != ctx) {
    // First call in this context (a new process, a cudaDeviceReset, or a
    // context the caller made current): device addresses from another
    // context are not valid here, so look everything up again.
    int major = 0, minor = 0, sms = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    s.status = nullptr;
    if (major != 10 || minor != 0) {
      s.ok = DSQ_ERR_UNSUPPORTED_DEVICE;
    } else {
      void *p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_status_word);
      if (e != cudaSuccess) {
        s.ctx = 0;
        return fail(DSQ_ERR_CUDA, "cudaGetSymbolAddress(status): %s", cudaGetErrorString(e));
      }
      s.status = static_cast<uint32_t *>(p);
      s.sms = sms;
      s.ok = DSQ_OK;
    }
    s.ctx = ctx;
  }
  if (s.ok != DSQ_OK)
    return fail(s.ok, "device %d is not a compute capability 10.0 (B200) device", dev);
  if (status_word) *status_word = s.status;
  if (num_sms) *num_sms = s.sms;
  return DSQ_OK;
}

int wait_ctl(WaitCtl *ctl, int *num_sms) {
  uint32_t *st = nullptr;
  int rc = device_ready(&st, num_sms);
  if (rc != DSQ_OK) return rc;
  ctl->status = st;
  ctl->limit_ns = g_wait_limit_ns.load();
  return DSQ_OK;
}

int set_smem_once(const void *kernel, int bytes, const char *what) {
  struct Entry {
    const void *k;
    uint64_t ctx;   // the attribute belongs to the context it was set in
    int bytes;
  };
  static std::mutex mu;
  static Entry done[256];
  static int n_done = 0;
  int dev = 0;
  uint64_t ctx = 0;
  const int rc = current_context(&dev, &ctx);
  if (rc != DSQ_OK) return rc;
  std::lock_guard<std::mutex> lk(mu);
  for (int i = 0; i < n_done; ++i)
    if (done[i].k == kernel && done[i].ctx == ctx && done[i].bytes >= bytes) return DSQ_OK;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return fail(DSQ_ERR_LAUNCH, "%s: shared-memory attribute: %s", what, cudaGetErrorString(e));
  for (int i = 0; i < n_done; ++i)
    if (done[i].k == kernel && done[i].ctx == ctx) {
      done[i].bytes = bytes;
      return DSQ_OK;
    }
  if (n_done < 256) done[n_done++] = Entry{kernel, ctx, bytes};
  return DSQ_OK;
}

int after_launch(const char *what, int n_kernels) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(DSQ_ERR_LAUNCH, "%s: launch failed: %s", what, cudaGetErrorString(e));
  g_launches.fetch_add(static_cast<uint64_t>(n_kernels));
  return DSQ_OK;
}

}  // namespace dsq

extern "C" {

size_t dsq_row_bytes(int type, int64_t K) {
  if (type == DSQ_Q8_0 && K > 0 && K % 32 == 0) return static_cast<size_t>(K / 32 * 34);
  if (type == DSQ_Q4_K && K > 0 && K % 256 == 0) return static_cast<size_t>(K / 256 * 144);
  return 0;
}

int dsq_device_status(void *stream) {
  uint32_t *st = nullptr;
  int rc = dsq::device_ready(&st, nullptr);
  if (rc != DSQ_OK) return rc;
  cudaError_t e = cudaStreamSynchronize(dsq::as_stream(stream));
  if (e != cudaSuccess) return dsq::fail(DSQ_ERR_CUDA, "stream sync: %s", cudaGetErrorString(e));
  uint32_t v = 0;
  e = cudaMemcpyFromSymbol(&v, dsq::g_status_word, sizeof(v));
  if (e != cudaSuccess) return dsq::fail(DSQ_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
  const uint32_t zero = 0;
  e = cudaMemcpyToSymbol(dsq::g_status_word, &zero, sizeof(zero));
  if (e != cudaSuccess) return dsq::fail(DSQ_ERR_CUDA, "status clear: %s", cudaGetErrorString(e));
  if (v & dsq::kStatusTimeout)
    return dsq::fail(DSQ_ERR_TIMEOUT, "a bounded device wait expired (status word 0x%x)", v);
  if (v & dsq::kStatusRange)
    return dsq::fail(DSQ_ERR_RANGE,
                     "a prefill weight block admits dequantized values outside the binary16 range "
                     "(status word 0x%x); the outputs that read it are inf or NaN",
                     v);
  return DSQ_OK;
}

const char *dsq_last_error(void) { return dsq::t_error; }

const char *dsq_version(void) { return "libdsq 0.1.0 (sm_100a)"; }

uint64_t dsq_launch_count(void) { return dsq::g_launches.load(); }

int dsq_test_set_wait_limit_ns(uint64_t ns) {
  dsq::g_wait_limit_ns.store(ns == UINT64_MAX ? 1000ull * 1000ull * 1000ull : ns);
  return DSQ_OK;
}

}  // extern "C"
