// gemm.h -- launch interfaces of the tcgen05 GEMM kernels.
//
//  * fused dequant-GEMM: D[mdim x tokens] = deq(W)-tile (MMA M = 128, built in
//    shared memory by dequant warps from packed NF4 codes) x activation-tile^T
//    (MMA N = token tile, loaded by TMA), persistent over (m-tile, token-tile,
//    k-split) work units, TMEM accumulators double-buffered.  Forward: the
//    A tile is deq(W) rows (K-major); backward dX: the A tile is deq(W)^T
//    (MN-major).  The rank-r LoRA up-projection is appended as extra k-steps
//    whose A operand is the LoRA weight and whose B operand is the (scaled)
//    rank-r activation.
//  The rank-r LoRA contractions (X A^T, dY B, dY^T (s X A^T), X^T (s dY B))
//  are in lora.cu.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "codec.h"

namespace qlora {

enum class FusedDir : int { kFwd = 0, kBwd = 1 };

struct FusedArgs {
  const uint8_t* codes;      // packed NF4 codes of W [nw, kw]
  const uint8_t* qabs;       // E4M3 block constants
  const float* c2;           // per-group second-level absmax
  const float* mean;         // per-tensor mean of the block constants
  const float* absf;         // fp32 block constants (no double quantization), else null
  int64_t nw, kw;            // W shape (out, in)
  int64_t m;                 // token rows
  const uint16_t* lora_w;    // fwd: LoRA B [nw, r]; bwd: LoRA A [r, kw] (bf16)
  int r;                     // LoRA rank (multiple of 8)
  int lora_steps;            // ceil(r / 64) extra k-steps (0 disables the LoRA term)
  uint16_t* out;             // bf16 output [m, ldo] (split == 1)
  float* out_acc;            // fp32 accumulation [m, ldo] (split > 1)
  int64_t ldo;               // fwd nw, bwd kw
  int64_t mdim;              // MMA-M extent: fwd nw, bwd kw
  int ksteps;                // main k-steps: contraction / 64 (rounded up)
  int m_tiles, t_tiles, splits;
  int m_group;               // m-tiles swept across all token tiles before the next group
  CodebookParam cb;
  uint32_t* err;             // device error flag
};

// Token tile of the fused kernel: 256 for prefill-shaped calls; the backward
// also takes 16 for decode-shaped calls (M <= 16).
// codes_map: the packed codes as uint8 [nw, kw/2], no swizzle, box {32, 128}
// (forward) or {64, 64} (backward).
cudaError_t launch_fused(FusedDir dir, int token_tile, const FusedArgs& args, const CUtensorMap& act,
                         const CUtensorMap& lora_act, const CUtensorMap& codes_map, int num_sms,
                         cudaStream_t stream);
// out[i * ld_out + j] = bf16(scale * in[i * ld_in + j]) for j < cols_in, 0 for
// cols_in <= j < cols_out (i < rows): the decode backward's split-K dX.  The
// grid is at most 8 CTAs of 256 threads per SM (num_sms: the device's SM count).
cudaError_t launch_convert_bf16(const float* in, int64_t rows, int64_t cols_in, int64_t ld_in,
                                int64_t cols_out, float scale, uint16_t* out, int64_t ld_out, int num_sms,
                                cudaStream_t stream);

// LoRA gradients for few tokens (M <= 16), fp32 throughout on CUDA cores:
//   dA[j, k] = s * sum_m G[m, j] X[m, k];   dB[n, j] = s * sum_m dY[m, n] XA[m, j]
cudaError_t launch_small_grads(const float* G, int64_t ld_g, const float* XA, int64_t ld_xa,
                               const uint16_t* X, const uint16_t* dY, int64_t M, int64_t rows,
                               int64_t cols, int r, float s, float* dA, float* dB, int num_sms,
                               cudaStream_t stream);

}  // namespace qlora
