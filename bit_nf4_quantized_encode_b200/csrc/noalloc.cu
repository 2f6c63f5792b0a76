// noalloc.cu -- a variant of qlora_quantize_nf4_dq that needs no caller-
// supplied work buffer and allocates nothing.
//
// Who needs it: callers that cannot obtain device memory at the moment they
// quantize -- for example a serving process that reserves all of its memory at
// start-up and forbids allocation afterwards, code running inside another
// framework's allocator or out-of-memory handler, or a loader that has no
// handle to an allocator at all.  The ordinary entry point asks the caller for
// a work buffer; this one takes its scratch (the per-block absmax values and
// the per-CTA partial sums of their mean) from a fixed array compiled into the
// library instead.
//
// The array is file-scope device memory: every GPU that loads the library
// holds it (kNoAllocScratchBytes) until the process exits.  All calls share
// it, so calls that may overlap on the GPU -- on different streams, or from
// different host threads -- race on it; order them on one stream.  Nothing in
// it must start at zero: each call writes every absmax value and every partial
// sum it later reads.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "codec.h"
#include "internal.h"
#include "nf4_tables.h"
#include "qlora.h"

namespace qlora {
namespace {

constexpr int64_t kNoAllocMaxBlocks = QLORA_NOALLOC_MAX_ELEMENTS / 64;
constexpr int kNoAllocPartials = 2048;                                   // encode grid cap
constexpr size_t kNoAllocC1Bytes = static_cast<size_t>(kNoAllocMaxBlocks) * sizeof(float);
constexpr size_t kNoAllocScratchBytes = kNoAllocC1Bytes + kNoAllocPartials * sizeof(double);

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_ptr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};

// Set-up, once per device, with that device current: the device address of
// the scratch array (its name is only a host-side stand-in in host code).
qlora_status scratch_for_current_device(void** ptr, int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QLORA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_ptr[dev]) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return QLORA_ERR_CUDA;
    if (major != 10 || minor != 0) return QLORA_ERR_UNSUPPORTED;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return QLORA_ERR_CUDA;
    g_num_sms[dev] = sms;
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  *num_sms = g_num_sms[dev];
  return QLORA_OK;
}

}  // namespace
}  // namespace qlora

using namespace qlora;

extern "C" qlora_status qlora_quantize_nf4_dq_noalloc(const uint16_t* W, const qlora_nf4_tensor* out,
                                                       qlora_stream_t stream) {
  // the descriptor checks of qlora_quantize_nf4_dq, in the same order, so the
  // same bad call gets the same status from both entry points
  qlora_status st = check_tensor(out);
  if (st != QLORA_OK) return st;
  const int64_t numel = out->rows * out->cols;
  if (numel == 0) return QLORA_OK;
  if (!W) return QLORA_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(W) & 15u) != 0) return QLORA_ERR_ALIGN;
  // in place of the work-buffer size check: the built-in scratch's limit
  if (numel > QLORA_NOALLOC_MAX_ELEMENTS) return QLORA_ERR_WORKSPACE;
  const Nf4Tables& tabs = level_tables(out->quant_type);
  if (!tabs.ok) return QLORA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  int num_sms = 0;
  st = scratch_for_current_device(&scratch, &num_sms);
  if (st != QLORA_OK) return st;
  const EncodeTables et = encode_tables(tabs);
  const bool dq = out->blocksize2 != 0;

  const int64_t nblocks = (numel + 63) / 64;
  // without double quantization the block absmax values are the output itself
  float* c1buf = dq ? static_cast<float*>(scratch) : out->absmax;
  double* partials = reinterpret_cast<double*>(static_cast<unsigned char*>(scratch) + kNoAllocC1Bytes);
  int grid = static_cast<int>((nblocks * 8 + 255) / 256);
  const int wave = num_sms * encode_ctas_per_sm();             // one wave of resident CTAs
  const int cap = wave < kNoAllocPartials ? wave : kNoAllocPartials;
  if (grid > cap) grid = cap;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (counted(launch_encode(W, numel, et, out->codes, c1buf, partials, grid, s)) != cudaSuccess)
    return QLORA_ERR_CUDA;
  if (!dq) return QLORA_OK;
  const int64_t ngroups = (nblocks + 255) / 256;
  int grid2 = static_cast<int>((ngroups + 7) / 8);
  if (grid2 > num_sms * 4) grid2 = num_sms * 4;
  if (grid2 < 1) grid2 = 1;
  if (counted(launch_double_quant(c1buf, nblocks, partials, grid, out->absmax_q, out->absmax_c2,
                                  out->absmax_mean, grid2, s)) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return QLORA_OK;
}
