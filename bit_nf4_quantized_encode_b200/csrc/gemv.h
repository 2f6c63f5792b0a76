// gemv.h -- launch interface of the decode-shaped (M <= 16) forward kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace qlora {

struct GemvArgs {
  const uint8_t* qabs;       // E4M3 block constants of W
  const float* c2;           // per-group second-level absmax
  const float* mean;         // per-tensor mean
  int64_t nw, kw;            // W shape (rows = out features, cols = in features)
  int64_t m;                 // token rows (<= 16)
  float* yacc;               // fp32 [m, nw] accumulator, zero on entry
  int* counters;             // [m_tiles] finished shares per tile, zero on entry
  const float* xa;           // X A^T, fp32 [m, ld_xa]
  int64_t ld_xa;
  const uint16_t* lora_b;    // LoRA B [nw, r] bf16
  int r;
  float s;                   // LoRA scale
  uint16_t* y;               // bf16 [m, nw] output
  int m_tiles;               // tiles of gemv_tile_rows() weight rows
  int steps;                 // 256-column steps per row
  float level[16];           // NF4 levels
  uint32_t* err;             // device error flag
};

int gemv_tile_rows();

// X A^T (fp32 [m, ld] and optionally [m, r] copy) for m <= 16 tokens, plus
// zeroing of zero_f[zero_n] and zero_i[zero_ni] for k_gemv.
cudaError_t launch_xa_small(const uint16_t* X, const uint16_t* A, int64_t m, int64_t kw, int r, float* xa,
                            int64_t ld, float* xa_out, float* zero_f, int64_t zero_n, int* zero_i,
                            int zero_ni, cudaStream_t stream);

// codes_map: packed codes as uint8 [nw, kw/2], box {128, 256}, 128-byte swizzle.
// x_map: X bf16 [m, kw], box {64, 16}, 128-byte swizzle.
cudaError_t launch_gemv(const GemvArgs& args, const CUtensorMap& codes_map, const CUtensorMap& x_map,
                        int num_sms, cudaStream_t stream);

}  // namespace qlora
