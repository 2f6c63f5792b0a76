// codec.h -- kernel-side parameter blocks and launchers of the NF4 codec.
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

namespace qlora {

// Bucketed decision table of the encoder, passed by value (kernel parameter).
// Buckets 33..63 are padding (never reached for finite inputs).
constexpr int kBuckets = 64;
struct EncodeTables {
  float bucket_thr[kBuckets];       // exact path: the threshold inside bucket u (or +inf)
  uint8_t bucket_base[kBuckets];    // exact path: code of the smallest n in bucket u
  uint32_t bucket_fast[kBuckets];   // fast path: threshold bits with base + 1 in the low 5 bits
  int fast;                         // nonzero: the reciprocal path may be used
};

// The 16 levels of the weight's 4-bit type, passed by value.
struct CodebookParam {
  float level[16];
};

// The codec kernels are launched as programmatic dependents of the kernel
// before them in the stream (each waits for it before touching global memory),
// so back-to-back calls overlap one launch's start with the previous one's end.
cudaError_t launch_encode(const uint16_t* w, int64_t numel, const EncodeTables& tab, uint8_t* codes,
                          float* c1buf, double* partials, int grid, cudaStream_t stream);
// Resident k_encode / k_dequant CTAs per SM (their grids are one wave of them).
int encode_ctas_per_sm();
int dequant_ctas_per_sm();
// k_double_quant is launched as the programmatic dependent of k_encode, which
// must be the kernel before it in the stream.
cudaError_t launch_double_quant(const float* c1buf, int64_t nblocks, const double* partials,
                                int npartials, uint8_t* q, float* c2, float* mean, int grid,
                                cudaStream_t stream);
// absf: the fp32 block constants of a weight stored without double
// quantization (qabs, c2 and mean are then unused), else NULL.
cudaError_t launch_dequant(const uint8_t* codes, const uint8_t* qabs, const float* c2,
                           const float* mean, const float* absf, int64_t numel, const CodebookParam& cb,
                           uint16_t* out, int grid, cudaStream_t stream);

}  // namespace qlora
