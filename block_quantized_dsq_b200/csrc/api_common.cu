// api_common.cu -- libdsq entry points that launch nothing (sizes, status,
// errors, version) and the host plumbing declared in dsq_host.h.
#include <atomic>
#include <cstdarg>
#include <cstring>
#include <mutex>

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

constexpr int kMaxDevices = 64;
std::mutex g_dev_mu;
struct DevState {
  bool checked = false;
  int ok = DSQ_ERR_UNSUPPORTED_DEVICE;
  uint32_t *status = nullptr;
  int sms = 0;
};
DevState g_dev[kMaxDevices];
}  // namespace

int fail(int code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_error, sizeof(t_error), fmt, ap);
  va_end(ap);
  return code;
}

int device_ready(uint32_t **status_word, int *num_sms) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(DSQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(DSQ_ERR_UNSUPPORTED_DEVICE, "device %d", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevState &s = g_dev[dev];
  if (!s.checked) {
    s.checked = true;
    int major = 0, minor = 0, sms = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (major != 10 || minor != 0) {
      s.ok = DSQ_ERR_UNSUPPORTED_DEVICE;
    } else {
      void *p = nullptr;
      e = cudaGetSymbolAddress(&p, g_status_word);
      if (e != cudaSuccess) {
        s.checked = false;
        return fail(DSQ_ERR_CUDA, "cudaGetSymbolAddress(status): %s", cudaGetErrorString(e));
      }
      s.status = static_cast<uint32_t *>(p);
      s.sms = sms;
      s.ok = DSQ_OK;
    }
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
    int dev;
    int bytes;
  };
  static std::mutex mu;
  static Entry done[256];
  static int n_done = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  for (int i = 0; i < n_done; ++i)
    if (done[i].k == kernel && done[i].dev == dev && done[i].bytes >= bytes) return DSQ_OK;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return fail(DSQ_ERR_LAUNCH, "%s: shared-memory attribute: %s", what, cudaGetErrorString(e));
  for (int i = 0; i < n_done; ++i)
    if (done[i].k == kernel && done[i].dev == dev) {
      done[i].bytes = bytes;
      return DSQ_OK;
    }
  if (n_done < 256) done[n_done++] = Entry{kernel, dev, bytes};
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
