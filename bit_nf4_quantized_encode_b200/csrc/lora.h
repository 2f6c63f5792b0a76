// lora.h -- launch interface of the rank-r contraction kernel (lora.cu): the
// LoRA branch's X A^T, dY B, dY^T (s X A^T) and X^T (s dY B).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace qlora {

// One contraction D[mdim, ndim] = P Q^T over `ksteps` 64-wide k-steps.  P is
// the long operand (tiles of 128 rows), Q the rank-r one (tiles of 64 rows,
// ndim = r); a_mn / b_mn: the operand is stored MN-major (the contraction
// index outermost) instead of K-major.
struct RankProblem {
  int64_t mdim, ndim;
  int ksteps;
  int m_tiles, n_tiles, splits;
  int unit_begin;            // first unit index of this problem in the launch
  int a_mn, b_mn;
  // outputs (either may be null)
  float* out_f32;            // D, or D^T when transpose; row stride ld_f32
  int64_t ld_f32;
  int transpose;
  uint16_t* out_bf16;        // bf16(bf16_scale * D) for columns < bf16_cols (zeros past ndim)
  int64_t ld_bf16;
  int64_t bf16_cols;         // a multiple of 64, <= 64 * n_tiles
  float bf16_scale;
  // split contraction (splits > 1): fp32 partial tiles and per-tile counters,
  // the counters zero before the launch
  float* slots;              // rank_slot_bytes(m_tiles * n_tiles, splits)
  uint32_t* counters;        // [m_tiles * n_tiles]
};

struct RankArgs {
  RankProblem p[2];
  int nprob;                 // 1 or 2
  int total_units;           // sum over problems of m_tiles * n_tiles * splits
  // side job: cvt_out[i, c] = bf16(cvt_scale * cvt_in[i, c]) for c < cvt_cols,
  // 0 for cvt_cols <= c < cvt_cols_out (a multiple of 8); cvt_in null: none
  const float* cvt_in;
  int64_t cvt_rows, cvt_cols, cvt_ld_in;
  uint16_t* cvt_out;
  int64_t cvt_ld_out, cvt_cols_out;
  float cvt_scale;
  uint32_t* err;
};

// K splits for `tiles` output tiles of `ksteps` k-steps: the count that
// minimises waves-of-units x k-steps-per-unit over num_sms SMs, with at least
// 4 k-steps per split and at most max(4, ceil(2 num_sms / tiles)) and
// max_splits splits.
int rank_splits(int tiles, int ksteps, int num_sms, int max_splits);
// Bytes of the partial-tile slots of a problem.
size_t rank_slot_bytes(int tiles, int splits);
// Tensor maps: am*/bm* of the problems' P and Q (bf16, 128B swizzle, box
// {64, 128} / {64, 64} K-major, {64, 64} MN-major); am1/bm1 unused when nprob == 1.
cudaError_t launch_rank(const RankArgs& args, const CUtensorMap& am0, const CUtensorMap& bm0,
                        const CUtensorMap& am1, const CUtensorMap& bm1, int num_sms, cudaStream_t stream);

}  // namespace qlora
