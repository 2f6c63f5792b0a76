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
//   Without double quantization the fp32 c1 is stored and used as the
//   constant (w' = bf16_RNE(L[code] * c1)); the levels L are those of the
//   weight's 4-bit type (NF4, or the FP4 / INT4 tables it is compared with).
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
// Lanes 4j..4j+3 of a warp own one 64-weight block, 16 consecutive weights per
// lane (two 16-byte loads, one 8-byte store of codes).  A CTA writes c1 per
// block and one double partial sum of c1 (for the tensor mean).  Full blocks
// go through the main loop; a ragged last block (numel not a multiple of 64)
// is encoded by one thread afterwards.
//
// Fast path: n' = RN(x * RN(1/c1)) is within 2^-22 of the IEEE quotient
// n = RN(x / c1) (three roundings of relative size 2^-24, |n| <= 1), so
// code(n) == code(n') unless a threshold lies within 2^-22 of n'.  The bucket
// of n' holds the only threshold that could (the table builder keeps every
// threshold 2^-18 away from the bucket edges); its fast-path word carries that
// threshold to within 2^-19 together with base + 1, and the code is
// base + 1 - [n' < thr'].  When any element of the lane lands within 2^-18 of
// its bucket's threshold (or is NaN), the lane redoes its 16 weights with IEEE
// divisions and the exact table.

constexpr float kRiskBand = 0x1.0p-18f;

// Exact code of n (float) from the exact bucket table.
__device__ __forceinline__ uint32_t exact_code(float n, const float* s_thr, const uint8_t* s_base) {
  const uint32_t u = __float_as_uint(__fmaf_rn(n, 16.0f, 8388624.0f)) & 63u;
  return s_base[u] + (n >= s_thr[u] ? 1u : 0u);
}

// Packed pairs of floats (sm_100 f32x2 arithmetic, round to nearest even;
// each lane of the pair rounds exactly as the scalar operation does).
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  uint64_t v;
  asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(lo), "f"(hi));
  return v;
}
__device__ __forceinline__ void unpack_f32x2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t sub_f32x2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// Per half: the larger of |a| and |b| as its magnitude (bf16 pairs).
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ float nan_min_abs(float m, float d) {
  float r;
  asm("{\n\t.reg .f32 t;\n\tabs.f32 t, %2;\n\tmin.NaN.f32 %0, %1, t;\n\t}" : "=f"(r) : "f"(m), "f"(d));
  return r;
}

__global__ void __launch_bounds__(256) k_encode(const uint16_t* __restrict__ w, int64_t numel,
                                                EncodeTables tab, uint8_t* __restrict__ codes,
                                                float* __restrict__ c1buf,
                                                double* __restrict__ partials) {
  __shared__ uint32_t s_fast[kBuckets];
  __shared__ float s_thr[kBuckets];
  __shared__ uint8_t s_base[kBuckets];
  __shared__ double s_red[8];
  for (int i = threadIdx.x; i < kBuckets; i += blockDim.x) {
    s_fast[i] = tab.bucket_fast[i];
    s_thr[i] = tab.bucket_thr[i];
    s_base[i] = tab.bucket_base[i];
  }
  __syncthreads();
  // launched as a programmatic dependent: the previous kernel in the stream may
  // still be running; nothing in global memory is read or written before it ends
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const uint32_t fast_tbl = static_cast<uint32_t>(__cvta_generic_to_shared(s_fast));
  const bool fast_ok = tab.fast != 0;

  const int64_t full_blocks = numel / 64;
  const int64_t nq = full_blocks * 4;               // lane tasks of 16 weights
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const uint4* w4 = reinterpret_cast<const uint4*>(w);
  double csum = 0.0;
  // One task: 16 weights already loaded (r0, r1); lanes 4j..4j+3 share a block.
  // Every lane executes the shuffles; `on` only gates the stores.
  auto task = [&](int64_t v, bool on, const uint4 r0, const uint4 r1) {
    const uint32_t wd[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
    float x[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      x[2 * k] = bf16_lo(wd[k]);
      x[2 * k + 1] = bf16_hi(wd[k]);
    }
    // |x| max on the packed pairs: the magnitude of max.xorsign.abs is the
    // larger magnitude, exactly (NaN weights are outside the encoder's domain)
    uint32_t pmax = 0u;
#pragma unroll
    for (int k = 0; k < 8; ++k) pmax = bf16x2_absmax(pmax, wd[k]);
    float amax = fmaxf(fabsf(bf16_lo(pmax)), fabsf(bf16_hi(pmax)));
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
    if (!on) return;

    uint32_t lo = 0x77777777u, hi = 0x77777777u;      // all zero-level codes
    if (amax > 0.0f) {
      // 1/c1 must be finite and c1 finite for the fast path
      bool exact = !fast_ok || !(amax >= 0x1.0p-125f) || !(amax <= 3.0e38f);
      if (!exact) {
        const float r = __frcp_rn(amax);
        const uint64_t r2 = pack_f32x2(r, r);
        const uint64_t c16 = pack_f32x2(16.0f, 16.0f), cbias = pack_f32x2(8388624.0f, 8388624.0f);
        float m = INFINITY;
        uint32_t pk[2] = {0u, 0u};
        // nibble order: element 2j -> high nibble of byte j; shift-add from byte 3 down.
        // The two elements of a word go through the same packed multiply, fma
        // and subtraction (each rounded like its scalar form).
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int jj = 3; jj >= 0; --jj) {
            const uint64_t n2 = mul_f32x2(pack_f32x2(x[8 * h + 2 * jj], x[8 * h + 2 * jj + 1]), r2);
            float f[2];
            unpack_f32x2(fma_f32x2(n2, c16, cbias), f[0], f[1]);
            uint32_t tw[2];
#pragma unroll
            for (int e = 0; e < 2; ++e)
              asm("ld.shared.b32 %0, [%1];" : "=r"(tw[e]) : "r"(fast_tbl + (__float_as_uint(f[e]) & 63u) * 4u));
            float d[2];
            unpack_f32x2(sub_f32x2(n2, pack_f32x2(__uint_as_float(tw[0]), __uint_as_float(tw[1]))), d[0], d[1]);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              m = nan_min_abs(m, d[e]);
              const uint32_t code = (tw[e] & 31u) - (__float_as_uint(d[e]) >> 31);
              pk[h] = (pk[h] << 4) + code;
            }
          }
        }
        if (!(m > kRiskBand)) exact = true;
        else { lo = pk[0]; hi = pk[1]; }
      }
      if (exact) {
        uint32_t pk[2] = {0u, 0u};
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int jj = 3; jj >= 0; --jj)
#pragma unroll
            for (int e = 0; e < 2; ++e)
              pk[h] = (pk[h] << 4) + exact_code(__fdiv_rn(x[8 * h + 2 * jj + e], amax), s_thr, s_base);
        lo = pk[0];
        hi = pk[1];
      }
    }
    reinterpret_cast<uint2*>(codes)[v] = make_uint2(lo, hi);
    if ((threadIdx.x & 3) == 0) {
      c1buf[v >> 2] = amax;
      csum += static_cast<double>(amax);
    }
  };
  // two tasks per iteration (a grid stride apart), both loaded before either is
  // encoded; the loop bound is uniform over the CTA, so every lane reaches the
  // shuffles
  for (int64_t b0 = static_cast<int64_t>(blockIdx.x) * blockDim.x; b0 < nq; b0 += 2 * stride) {
    const int64_t v0 = b0 + threadIdx.x, v1 = v0 + stride;
    const bool on0 = v0 < nq, on1 = v1 < nq;
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    uint4 a0 = z, a1 = z, c0 = z, c1 = z;
    if (on0) { a0 = __ldg(w4 + 2 * v0); a1 = __ldg(w4 + 2 * v0 + 1); }
    if (on1) { c0 = __ldg(w4 + 2 * v1); c1 = __ldg(w4 + 2 * v1 + 1); }
    task(v0, on0, a0, a1);
    if (b0 + stride < nq) task(v1, on1, c0, c1);      // uniform over the CTA
  }
  // k_double_quant (launched as this grid's programmatic dependent) may now be
  // scheduled; it waits for the whole grid before reading anything
  asm volatile("griddepcontrol.launch_dependents;");
  // ragged last block: one thread, exact path
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0 && full_blocks * 64 < numel) {
    const int64_t e0 = full_blocks * 64;
    float amax = 0.0f;
    for (int64_t e = e0; e < numel; ++e)
      amax = fmaxf(amax, fabsf(__uint_as_float(static_cast<uint32_t>(w[e]) << 16)));
    const int64_t nbytes = (numel + 1) / 2;
    for (int64_t j = e0 / 2; j < nbytes; ++j) {
      uint32_t c[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int64_t idx = 2 * j + e;
        c[e] = 7u;
        if (idx < numel && amax > 0.0f)
          c[e] = exact_code(__fdiv_rn(__uint_as_float(static_cast<uint32_t>(w[idx]) << 16), amax), s_thr, s_base);
      }
      codes[j] = static_cast<uint8_t>((c[0] << 4) | c[1]);
    }
    c1buf[full_blocks] = amax;
    csum += static_cast<double>(amax);
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
  asm volatile("griddepcontrol.wait;" ::: "memory");   // k_encode complete
  asm volatile("griddepcontrol.launch_dependents;");   // a dependent waits for this grid itself
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
// One lane per 32 codes (16 bytes in, 64 bytes out); a 64-weight block is two
// lanes.  Each lane takes kDqUnroll chunks per iteration (a grid stride apart)
// and issues the loads of all of them before expanding any: with two CTAs per
// SM that keeps about 64 KB of codes in flight per SM, above HBM's
// bandwidth-delay product.  A ragged last chunk is expanded element by element.
constexpr int kDqUnroll = 8;
// c2v is the group's c2 with double quantization, the block's own fp32
// constant without it (plain).
__device__ __forceinline__ void dequant_chunk(const uint4 cw, uint32_t q, float c2v, float mu, bool plain,
                                              const CodebookParam& cb, uint4 (&o)[4]) {
  const float c1p = plain ? c2v : block_constant(q, __fdiv_rn(c2v, 448.0f), mu);
  const ByteTables t = make_tables(cb.level, c1p);
  o[0] = expand8(cw.x, t);
  o[1] = expand8(cw.y, t);
  o[2] = expand8(cw.z, t);
  o[3] = expand8(cw.w, t);
}

// The 32 lanes of a warp expand 32 consecutive chunks (2 KB of output).  Each
// lane parks its 64 bytes in shared memory (rows of 80 bytes: conflict-free),
// then the warp stores the 2 KB with every instruction covering 512
// contiguous bytes.
__global__ void __launch_bounds__(256) k_dequant(const uint8_t* __restrict__ codes,
                                                 const uint8_t* __restrict__ qabs,
                                                 const float* __restrict__ c2, const float* __restrict__ mean,
                                                 const float* __restrict__ absf, int64_t numel,
                                                 CodebookParam cb, uint16_t* __restrict__ out) {
  __shared__ __align__(16) uint8_t s_out[8][32 * 80];
  // a programmatic dependent of the previous kernel in the stream: wait for it
  // before touching global memory, then let the next one launch
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  const bool plain = absf != nullptr;                // fp32 block constants, no double quantization
  const float mu = plain ? 0.0f : __ldg(mean);
  const int64_t nfull = numel / 32;                  // chunks of 32 real weights
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const uint4* cw4 = reinterpret_cast<const uint4*>(codes);
  uint4* out4 = reinterpret_cast<uint4*>(out);
  const int lane = threadIdx.x & 31;
  uint8_t* st = s_out[threadIdx.x >> 5];
  // the loop bound is uniform over the CTA, so every lane reaches the syncwarps
  for (int64_t b0 = static_cast<int64_t>(blockIdx.x) * blockDim.x; b0 < nfull; b0 += kDqUnroll * stride) {
    const int64_t ch = b0 + threadIdx.x;
    uint4 cw[kDqUnroll];
    uint32_t qv[kDqUnroll];
    float c2v[kDqUnroll];
#pragma unroll
    for (int u = 0; u < kDqUnroll; ++u) {
      const int64_t c = ch + u * stride;
      cw[u] = make_uint4(0u, 0u, 0u, 0u);
      qv[u] = 0;
      c2v[u] = 0.0f;
      if (c < nfull) {
        cw[u] = __ldg(cw4 + c);
        if (plain) {
          c2v[u] = __ldg(absf + (c >> 1));
        } else {
          qv[u] = __ldg(qabs + (c >> 1));
          c2v[u] = __ldg(c2 + (c >> 9));
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kDqUnroll; ++u) {
      const int64_t c = ch + u * stride;
      const int64_t wc0 = c - lane;                  // the warp's first chunk
      uint4 o[4];
      dequant_chunk(cw[u], qv[u], c2v[u], mu, plain, cb, o);
#pragma unroll
      for (int k = 0; k < 4; ++k) *reinterpret_cast<uint4*>(st + lane * 80 + k * 16) = o[k];
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int p = lane + 32 * j;                 // 16-byte piece of the warp's 2 KB
        const int src = p >> 2;                      // the lane that expanded it
        if (wc0 + src < nfull) out4[wc0 * 4 + p] = *reinterpret_cast<const uint4*>(st + src * 80 + (p & 3) * 16);
      }
      __syncwarp();
    }
  }
  // ragged last chunk
  if (blockIdx.x == 0 && threadIdx.x == 0 && nfull * 32 < numel) {
    const int64_t blk = nfull >> 1;
    const float c1p = plain ? absf[blk] : block_constant(qabs[blk], __fdiv_rn(c2[blk >> 8], 448.0f), mu);
    for (int64_t e = nfull * 32; e < numel; ++e) {
      const uint32_t byte = codes[e >> 1];
      const uint32_t code = (e & 1) ? (byte & 15u) : (byte >> 4);
      const __nv_bfloat16 v = __float2bfloat16_rn(__fmul_rn(cb.level[code], c1p));
      out[e] = *reinterpret_cast<const uint16_t*>(&v);
    }
  }
}

// ------------------------------------------------------------------ launchers
// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel in the stream finishes (it waits for that kernel
// with griddepcontrol.wait before using global memory).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), int grid, cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

cudaError_t launch_encode(const uint16_t* w, int64_t numel, const EncodeTables& tab, uint8_t* codes,
                          float* c1buf, double* partials, int grid, cudaStream_t stream) {
  return launch_pdl(k_encode, grid, stream, w, numel, tab, codes, c1buf, partials);
}

cudaError_t launch_double_quant(const float* c1buf, int64_t nblocks, const double* partials,
                                int npartials, uint8_t* q, float* c2, float* mean, int grid,
                                cudaStream_t stream) {
  // programmatic dependent of k_encode: the launch overlaps the encoder's tail
  return launch_pdl(k_double_quant, grid, stream, c1buf, nblocks, partials, npartials, q, c2, mean);
}

int dequant_ctas_per_sm() {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_dequant, 256, 0) != cudaSuccess || n < 1) n = 1;
  return n;
}

int encode_ctas_per_sm() {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_encode, 256, 0) != cudaSuccess || n < 1) n = 1;
  return n;
}

cudaError_t launch_dequant(const uint8_t* codes, const uint8_t* qabs, const float* c2,
                           const float* mean, const float* absf, int64_t numel, const CodebookParam& cb,
                           uint16_t* out, int grid, cudaStream_t stream) {
  return launch_pdl(k_dequant, grid, stream, codes, qabs, c2, mean, absf, numel, cb, out);
}

}  // namespace qlora
