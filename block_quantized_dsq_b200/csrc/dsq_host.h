// dsq_host.h -- host-side plumbing shared by the libdsq entry points:
// per-thread error text, argument checks, the per-device status word and the
// launch counter.
#pragma once

#include <cstdint>
#include <cstdio>
#include <utility>
#include <cuda_runtime.h>

#include "../../include/dsq.h"
#include "dsq_device.cuh"

namespace dsq {

// Records a message for dsq_last_error() and returns `code`.
int fail(int code, const char *fmt, ...);

constexpr int kMaxDevices = 64;

// The current device and a process-unique id of the CUDA context current on
// this thread (never reused, never 0).  Caches of device addresses or
// per-context settings are keyed by this id, so none outlives its context
// (cudaDeviceReset, or a driver context the caller made current).
int current_context(int *device, uint64_t *ctx_id);

// Checks the current device once per context (compute capability 10.0) and
// returns its status-word pointer and SM count through the out-parameters.
int device_ready(uint32_t **status_word, int *num_sms);

// Wait control for kernels launched now (status word + current limit).
int wait_ctl(WaitCtl *ctl, int *num_sms);

// After a launch: maps a launch error to DSQ_ERR_LAUNCH and counts launches.
int after_launch(const char *what, int n_kernels = 1);

// One token of a single weight through the multi-token GEMV (gemv_tokens.cu),
// errors named after `name`.
int gemv_one_token(const char *name, int type, const void *w, int64_t N, int64_t K, const int8_t *xq,
                   const float *xd, const int32_t *xs, float *y, cudaStream_t stream);

// Raises a kernel's dynamic shared-memory limit once per (kernel, context):
// the first call in a context configures it; later calls (for example inside
// a CUDA graph capture) only launch.
int set_smem_once(const void *kernel, int bytes, const char *what);

// Launches `kern` on `stream` with programmatic stream serialization, so it
// may start before the previous kernel on the stream has finished (the
// kernel itself orders its dependent accesses with pdl_wait()).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

inline bool aligned(const void *p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

inline cudaStream_t as_stream(void *s) { return static_cast<cudaStream_t>(s); }

}  // namespace dsq

#define DSQ_REQUIRE(cond, code, ...)              \
  do {                                            \
    if (!(cond)) return ::dsq::fail((code), __VA_ARGS__); \
  } while (0)
