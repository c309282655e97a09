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
#include <algorithm>
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

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

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
  // Same scratch layout as gpt2_op_lmhead_ce: partials [groups][M] float2,
  // target logits [M], per-position losses [M].
  const size_t groups = lmhead_groups_max(V);
  const size_t part_bytes = align256(groups * (size_t)M * sizeof(float2));
  const size_t need = part_bytes + 2 * align256((size_t)M * 4);
  if (need > (size_t)GPT2_NOALLOC_SCRATCH_BYTES) return GPT2_ERR_SCRATCH_LIMIT;

  NoallocDevice* d = nullptr;
  int rc = noalloc_setup(&d);
  if (rc != GPT2_OK) return rc;
  uint8_t* ws = static_cast<uint8_t*>(d->scratch);
  float2* part = reinterpret_cast<float2*>(ws);
  float* tgt = reinterpret_cast<float*>(ws + part_bytes);
  float* tok = reinterpret_cast<float*>(ws + part_bytes + align256((size_t)M * 4));
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  GemmArgs a{};
  a.M = M;
  a.N = V;
  a.K = C;
  a.out = logits_or_null;
  a.ldo = V;
  a.targets = targets;
  a.part = part;
  a.tgt_logit = tgt;
  a.status = status;
  int n_groups;
  if (dtype == GPT2_BF16) {
    const int bn = std::max(gemm_tc_pick_bn(M, V, d->num_sms, EPI_LMHEAD), LMHEAD_MIN_BN);
    n_groups = gemm_tc_n_tiles(V, bn);
    CUtensorMap ta, tb;
    if (!make_tmap_bf16(&ta, hf, M, C, C, 128) || !make_tmap_bf16(&tb, wte, V, C, C, bn)) return GPT2_ERR_CUDA;
    if (gemm_tc_launch(EPI_LMHEAD, bn, ta, tb, ta, a, d->num_sms, s) != cudaSuccess) return GPT2_ERR_CUDA;
  } else {
    n_groups = (V + SIMT_BN - 1) / SIMT_BN;
    if (gemm_simt_launch(EPI_LMHEAD, static_cast<const float*>(hf), static_cast<const float*>(wte), a, s) !=
        cudaSuccess)
      return GPT2_ERR_CUDA;
  }
  return ce_finish_launch(part, n_groups, tgt, targets, M, V, token_loss_or_null ? token_loss_or_null : tok, loss_out,
                          status, s) == cudaSuccess
             ? GPT2_OK
             : GPT2_ERR_CUDA;
}
