// codec.cu -- blockwise NF4 encode, double quantization of the block
// constants, and two-level dequantization to bf16 (sm_100a).
//
// Method (QLoRA, arXiv:2305.14314, as summarised by automatone "QLoRA paper
// explained", paragraphs "4-bit NormalFloat (NF4)" and "Double Quantization
// (DQ)", and creativeworksofknowledge "QLoRA: Fine-Tune 70B on One GPU",
// sections "1. NF4" and "2. Double quantization"):
//   per 64 weights  c1 = max |x|;  n = x / c1 (IEEE float division);
//                   code = nearest NF4 level, ties to the lower index;
//                   byte j of the packed stream = code[2j] << 4 | code[2j+1].
//   per tensor      mu = float(double-sum(c1) / nblocks);
//   per 256 c1      c2 = max |c1 - mu|;  q = E4M3_RNE(float((c1-mu)/c2) * 448), 0 if c2 == 0.
//   dequant         c1' = fma(e4m3(q), c2/448, mu);  w' = bf16_RNE(L[code] * c1').
// Every float operation uses an explicitly rounded intrinsic so the compiler
// cannot contract or reorder it: the results are bit-identical to any
// implementation that performs the same IEEE operations.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "codec.h"
#include "nf4_device.cuh"

namespace qlora {

// ------------------------------------------------------------------ encode
// One thread per 8 consecutive weights (one 16-byte load); 8 lanes form one
// 64-weight block.  Writes packed codes, c1 per block, and one double partial
// sum of c1 per CTA (for the tensor mean).  All 32 lanes of a warp execute
// every shuffle; `mode` only changes how a lane loads and stores.
enum : int { kVecNone = 0, kVecFull = 1, kVecTail = 2 };

__device__ __forceinline__ void encode_vec(const uint16_t* __restrict__ w, int64_t numel,
                                           int64_t v, int mode, bool fast, const float* s_thr,
                                           const uint8_t* s_base, uint8_t* __restrict__ codes,
                                           float* __restrict__ c1buf, double& csum) {
  float x[8];
  const int64_t e0 = v * 8;
  if (mode == kVecFull) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(w) + v);
    x[0] = bf16_lo(raw.x); x[1] = bf16_hi(raw.x); x[2] = bf16_lo(raw.y); x[3] = bf16_hi(raw.y);
    x[4] = bf16_lo(raw.z); x[5] = bf16_hi(raw.z); x[6] = bf16_lo(raw.w); x[7] = bf16_hi(raw.w);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      x[i] = (mode == kVecTail && e0 + i < numel)
                 ? __uint_as_float(static_cast<uint32_t>(w[e0 + i]) << 16) : 0.0f;
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(x[i]));
  // reduce over the 8 lanes of this block (lanes 8j..8j+7 of the warp)
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 4));
  if (mode == kVecNone) return;

  uint32_t packed = 0x77777777u;          // all zero-level codes
  if (amax > 0.0f) {
    // Fast path: n' = RN(x * RN(1/c1)) is within 2^-22 of the IEEE quotient
    // RN(x / c1) (three roundings of relative size 2^-24, |n| <= 1), so its
    // code equals the quotient's unless a threshold lies within 2^-22 of n'.
    // The bucket of n' holds the only threshold that close (the table check
    // keeps every threshold 2^-20 away from bucket edges); when n' is within
    // 2^-20 of it the block's vector is redone with IEEE divisions.
    bool exact = !fast || amax < 0x1.0p-125f;       // 1 / c1 must stay finite
    if (!exact) {
      const float r = __frcp_rn(amax);
      uint32_t pk = 0;
      bool risky = false;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float n = __fmul_rn(x[i], r);
        const uint32_t u = __float_as_uint(__fmaf_rn(n, 16.0f, 8388624.0f)) & 63u;
        const float d = __fsub_rn(n, s_thr[u]);     // exact sign; -inf when the bucket has no threshold
        uint32_t code = s_base[u] + (d >= 0.0f ? 1u : 0u);
        risky |= fabsf(d) <= 0x1.0p-20f;
        if (mode == kVecTail && e0 + i >= numel) code = 7u;
        pk |= code << (8 * (i >> 1) + ((i & 1) ? 0 : 4));
      }
      if (risky) exact = true;
      else packed = pk;
    }
    if (exact) {
      packed = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float n = __fdiv_rn(x[i], amax);
        // bucket u = RN(16 n + 16) via one fma against 2^23; then one compare
        const uint32_t u = __float_as_uint(__fmaf_rn(n, 16.0f, 8388624.0f)) & 63u;
        uint32_t code = s_base[u] + (n >= s_thr[u] ? 1u : 0u);
        if (mode == kVecTail && e0 + i >= numel) code = 7u;
        // element 2j -> high nibble of byte j, element 2j+1 -> low nibble
        packed |= code << (8 * (i >> 1) + ((i & 1) ? 0 : 4));
      }
    }
  }
  if (mode == kVecFull) {
    reinterpret_cast<uint32_t*>(codes)[v] = packed;
  } else {
    const int64_t nbytes = (numel + 1) / 2;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (v * 4 + j < nbytes) codes[v * 4 + j] = static_cast<uint8_t>(packed >> (8 * j));
  }
  if ((threadIdx.x & 7) == 0) {
    c1buf[v >> 3] = amax;
    csum += static_cast<double>(amax);
  }
}

__global__ void __launch_bounds__(256) k_encode(const uint16_t* __restrict__ w, int64_t numel,
                                                EncodeTables tab, uint8_t* __restrict__ codes,
                                                float* __restrict__ c1buf,
                                                double* __restrict__ partials) {
  __shared__ float s_thr[kBuckets];
  __shared__ uint8_t s_base[kBuckets];
  __shared__ double s_red[8];
  for (int i = threadIdx.x; i < kBuckets; i += blockDim.x) {
    s_thr[i] = tab.bucket_thr[i];
    s_base[i] = tab.bucket_base[i];
  }
  __syncthreads();

  // Vectors of 8 weights; a block of 64 is 8 vectors, i.e. 8 consecutive
  // threads of one warp (the CTA size and grid stride are multiples of 8).
  const int64_t nblocks = (numel + 63) / 64;
  const int64_t nvec = nblocks * 8;                 // padded to whole blocks
  const int64_t full_blocks = numel / 64;           // blocks with 64 real weights
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  double csum = 0.0;
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x; base < nvec; base += stride) {
    const int64_t v = base + threadIdx.x;
    const int64_t blk = v >> 3;                     // the same for all 8 lanes of a group
    const int mode = (blk < full_blocks) ? kVecFull : (blk < nblocks ? kVecTail : kVecNone);
    encode_vec(w, numel, v, mode, tab.fast != 0, s_thr, s_base, codes, c1buf, csum);
  }
  // deterministic per-CTA reduction of the partial sums
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) csum += __shfl_xor_sync(0xFFFFFFFFu, csum, o);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = csum;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) t += s_red[i];
    partials[blockIdx.x] = t;
  }
}

// ------------------------------------------------------------------ double quant
// Every CTA first reduces the per-CTA partial sums in the same fixed order
// (so all CTAs agree on mu), then one warp handles one group of 256 c1.
__global__ void __launch_bounds__(256) k_double_quant(const float* __restrict__ c1buf,
                                                      int64_t nblocks, const double* __restrict__ partials,
                                                      int npartials, uint8_t* __restrict__ q,
                                                      float* __restrict__ c2, float* __restrict__ mean_out) {
  __shared__ double s_red[256];
  double t = 0.0;
  for (int i = threadIdx.x; i < npartials; i += blockDim.x) t += partials[i];
  s_red[threadIdx.x] = t;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) s_red[threadIdx.x] += s_red[threadIdx.x + o];
    __syncthreads();
  }
  const float mu = __double2float_rn(__ddiv_rn(s_red[0], static_cast<double>(nblocks)));
  if (blockIdx.x == 0 && threadIdx.x == 0) *mean_out = mu;

  const int lane = threadIdx.x & 31;
  const int64_t ngroups = (nblocks + 255) / 256;
  const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       g < ngroups; g += warps_total) {
    const int64_t b0 = g * 256 + lane * 8;        // this lane's 8 constants
    float c[8];
    float dmax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      c[i] = (b0 + i < nblocks) ? c1buf[b0 + i] : mu;
      dmax = fmaxf(dmax, fabsf(__fsub_rn(c[i], mu)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dmax = fmaxf(dmax, __shfl_xor_sync(0xFFFFFFFFu, dmax, o));
    if (lane == 0) c2[g] = dmax;
    uint8_t qb[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint8_t v = 0;
      if (dmax > 0.0f) {
        const float tq = __fdiv_rn(__fsub_rn(c[i], mu), dmax);
        v = static_cast<uint8_t>(__nv_cvt_float_to_fp8(__fmul_rn(tq, 448.0f), __NV_SATFINITE, __NV_E4M3));
      }
      qb[i] = v;
    }
    if (b0 + 8 <= nblocks) {
      uint2 pk;
      pk.x = qb[0] | (qb[1] << 8) | (qb[2] << 16) | (static_cast<uint32_t>(qb[3]) << 24);
      pk.y = qb[4] | (qb[5] << 8) | (qb[6] << 16) | (static_cast<uint32_t>(qb[7]) << 24);
      *reinterpret_cast<uint2*>(q + b0) = pk;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (b0 + i < nblocks) q[b0 + i] = qb[i];
    }
  }
}

// ------------------------------------------------------------------ dequant
// One thread per 32 codes (16 bytes in, 64 bytes out); a 64-weight block is
// two threads.  Ragged tails fall back to element-wise work.
__global__ void __launch_bounds__(256) k_dequant(const uint8_t* __restrict__ codes,
                                                 const uint8_t* __restrict__ qabs,
                                                 const float* __restrict__ c2, const float* __restrict__ mean,
                                                 int64_t numel, CodebookParam cb,
                                                 uint16_t* __restrict__ out) {
  const float mu = __ldg(mean);
  const int64_t nchunks = (numel + 31) / 32;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t ch = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; ch < nchunks;
       ch += stride) {
    const int64_t blk = ch >> 1;
    const float c2v = __ldg(c2 + (blk >> 8));
    const float c1p = block_constant(__ldg(qabs + blk), __fdiv_rn(c2v, 448.0f), mu);
    const ByteTables t = make_tables(cb.level, c1p);
    const int64_t e0 = ch * 32;
    if (e0 + 32 <= numel) {
      const uint4 cw = __ldg(reinterpret_cast<const uint4*>(codes) + ch);
      uint4* dst = reinterpret_cast<uint4*>(out + e0);
      dst[0] = expand8(cw.x, t);
      dst[1] = expand8(cw.y, t);
      dst[2] = expand8(cw.z, t);
      dst[3] = expand8(cw.w, t);
    } else {
      for (int64_t e = e0; e < numel; ++e) {
        const uint32_t byte = codes[e >> 1];
        const uint32_t code = (e & 1) ? (byte & 15u) : (byte >> 4);
        const __nv_bfloat16 v = __float2bfloat16_rn(__fmul_rn(cb.level[code], c1p));
        out[e] = *reinterpret_cast<const uint16_t*>(&v);
      }
    }
  }
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_encode(const uint16_t* w, int64_t numel, const EncodeTables& tab, uint8_t* codes,
                          float* c1buf, double* partials, int grid, cudaStream_t stream) {
  k_encode<<<grid, 256, 0, stream>>>(w, numel, tab, codes, c1buf, partials);
  return cudaGetLastError();
}

cudaError_t launch_double_quant(const float* c1buf, int64_t nblocks, const double* partials,
                                int npartials, uint8_t* q, float* c2, float* mean, int grid,
                                cudaStream_t stream) {
  k_double_quant<<<grid, 256, 0, stream>>>(c1buf, nblocks, partials, npartials, q, c2, mean);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t* codes, const uint8_t* qabs, const float* c2,
                           const float* mean, int64_t numel, const CodebookParam& cb, uint16_t* out,
                           int grid, cudaStream_t stream) {
  k_dequant<<<grid, 256, 0, stream>>>(codes, qabs, c2, mean, numel, cb, out);
  return cudaGetLastError();
}

}  // namespace qlora
