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
  const float* absf;         // fp32 block constants (no double quantization), else null
  int64_t nw, kw;            // W shape (rows = out features, cols = in features)
  int64_t m;                 // token rows (<= 16)
  float* slots;              // fp32 [gemv_slot_floats()] partials of shared tiles
  uint32_t* cnt;             // [m_tiles * 8] per-warp tile counters, zeroed by k_xa_zero
  const float* xa_part;      // k_xa_zero's X A^T slices: [xa_splits][16][ld_xa] fp32
  int64_t ld_xa;             // 64 lora_steps
  int r;                     // LoRA rank (a multiple of 8)
  int lora_steps;            // 64-column groups of the rank
  int xa_splits;
  float s;                   // LoRA scale alpha / r
  const uint16_t* lora_b;    // B bf16 [nw, r] (with adapter_idx: [n_adapters][nw, r])
  const int32_t* adapter_idx;  // per-token adapter [m], or null for the single adapter
  int n_adapters;
  int64_t b_stride;          // elements between consecutive adapters' B (nw * r)
  uint16_t* y;               // Y bf16 [m, nw]
  float* xa_out;             // X A^T fp32 [m, r], or null
  int m_tiles;               // tiles of gemv_tile_rows() weight rows
  int steps;                 // 256-column steps per row
  float level[16];           // levels of the weight's 4-bit type
  uint32_t* err;             // device error flag
};

int gemv_tile_rows();
// At most this many k_gemv CTAs (one per SM on a B200).
constexpr int kMaxGemvCtas = 256;
// fp32 floats of k_gemv's partial slots for a weight of m_tiles x steps units.
int64_t gemv_slot_floats(int64_t m_tiles, int64_t steps);

// Upper bound on the K slices of X A^T (the work buffer holds that many).
constexpr int kMaxXaSplits = 16;
// K slices of X A^T for rank r and contraction kw (1 .. kMaxXaSplits).
int xa_splits_for(int r, int64_t kw);
// Partial X A^T (fp32 [splits][16][ld]) for m <= 16 tokens, and the zeroing of
// zero[n_zero] (k_gemv's tile counters; n_zero a multiple of 4, 16-byte aligned).
// With adapter_idx (device [m]), token i uses A + adapter_idx[i] * a_stride
// (A holds n_adapters adapters); a negative index gives that token X A^T = 0,
// and an index >= n_adapters does too and sets kErrBadAdapter in *err.
cudaError_t launch_xa_zero(const uint16_t* X, const uint16_t* A, int64_t m, int64_t kw, int r, float* part,
                           int64_t ld, int splits, float* zero, int64_t n_zero, const int32_t* adapter_idx,
                           int n_adapters, int64_t a_stride, uint32_t* err, cudaStream_t stream);

// codes_map: packed codes as uint8 [nw, kw/2], box {128, 256}, 128-byte swizzle.
// x_map: X bf16 [m, kw], box {64, m}, 128-byte swizzle.
// k_gemv is launched as a programmatic dependent of the kernel before it in the
// stream, which must be k_xa_zero of the same call; it writes Y (and X A^T).
cudaError_t launch_gemv(const GemvArgs& args, const CUtensorMap& codes_map, const CUtensorMap& x_map,
                        int num_sms, cudaStream_t stream);

}  // namespace qlora
