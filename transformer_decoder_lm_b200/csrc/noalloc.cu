// noalloc.cu - allocation-free variant of the lm_head + cross-entropy step.
//
// gpt2_op_lmhead_ce needs scratch memory for its per-row log-sum-exp
// partials, and takes it from a caller-provided workspace. Some callers have
// no way to provide one: code that runs inside a host application which owns
// every device allocation and forbids extra cudaMalloc calls (an inference
// server's plugin, a library embedded in another runtime's memory pool), or
// code on a latency-critical path where cudaMalloc's implicit device
// synchronisation is not acceptable. gpt2_op_lmhead_ce_noalloc serves them:
// its scratch is a fixed array in the library's own device image, so the
// call allocates nothing. The caller still owns and passes every input and
// output buffer.
//
// The array, g2_noalloc_scratch, holds GPT2_NOALLOC_SCRATCH_BYTES on every
// GPU that loads the library, for as long as the library stays loaded.
// Requests that would need more are rejected with GPT2_ERR_SCRATCH_LIMIT.
// Every call uses the same array, so calls whose kernels overlap on the GPU
// (on different streams, or from different host threads) race on it; keep
// them ordered. Nothing in the array has to start at zero: every partial
// that the finishing kernel reads is written earlier in the same call.
#include <mutex>

#include "common.cuh"
#include "gpt2.h"
#include "kernels.h"

namespace {

static __device__ __align__(256) unsigned char g2_noalloc_scratch[GPT2_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

struct NoallocDevice {
  bool ready = false;
  void* scratch = nullptr;   // device address of g2_noalloc_scratch on this device
  int num_sms = 0;
};

std::mutex g_mu;
NoallocDevice g_devices[kMaxDevices];


// Per-device set-up, done by the first call on each device with that device
// current: the scratch array's device address, the SM count and the GEMM
// kernels' shared-memory attribute.
int noalloc_setup(NoallocDevice** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GPT2_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  NoallocDevice& d = g_devices[dev];
  if (!d.ready) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g2_noalloc_scratch) != cudaSuccess || ptr == nullptr) return GPT2_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
      return GPT2_ERR_CUDA;
    if (g2::gemm_tc_set_attributes() != cudaSuccess) return GPT2_ERR_CUDA;
    d.scratch = ptr;
    d.num_sms = sms;
    d.ready = true;
  }
  *out = &d;
  return GPT2_OK;
}

}  // namespace

extern "C" int gpt2_op_lmhead_ce_noalloc(int dtype, const void* hf, const void* wte, const int32_t* targets, int M,
                                         int C, int V, float* logits_or_null, float* token_loss_or_null,
                                         float* loss_out, int* status, void* stream) {
  using namespace g2;
  if ((dtype != GPT2_BF16 && dtype != GPT2_FP32) || !hf || !wte || !targets || M < 1 || C < 8 || (C % 8) || V < 1 ||
      (reinterpret_cast<uintptr_t>(hf) & 15) || (reinterpret_cast<uintptr_t>(wte) & 15))
    return GPT2_ERR_INVALID_ARG;
  if (dtype == GPT2_BF16 && (C % 64)) return GPT2_ERR_UNSUPPORTED;
  // the same scratch layout and launches as gpt2_op_lmhead_ce
  if (lmhead_ce_scratch_bytes(M, V) > (size_t)GPT2_NOALLOC_SCRATCH_BYTES) return GPT2_ERR_SCRATCH_LIMIT;
  NoallocDevice* d = nullptr;
  const int rc = noalloc_setup(&d);
  if (rc != GPT2_OK) return rc;
  return lmhead_ce_launch(dtype == GPT2_BF16, hf, wte, targets, M, C, V, logits_or_null, token_loss_or_null, loss_out,
                          d->scratch, d->num_sms, status, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? GPT2_OK
             : GPT2_ERR_CUDA;
}
