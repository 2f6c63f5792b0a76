// gemv.cu -- decode-shaped forward of the NF4 LoRA linear layer (M <= 16 tokens).
//
// Y = X deq(W)^T + s (X A^T) B^T with few token rows is a stream over the packed
// weight (automatone "QLoRA paper explained", section "How it works": the 4-bit
// weight is dequantized on the fly for the matmul), bound by HBM.  Two kernels:
//
// k_xa_small: X A^T in fp32 on CUDA cores (one CTA per LoRA rank column); also
//   zeroes the split buffer and tile counters of k_gemv.
//
// k_gemv: the weight stream.  Each CTA takes an equal, contiguous share of all
//   (256-row tile, 256-column step) pairs, so the work is balanced whatever the
//   shape (a tile split between CTAs is combined with fp32 atomics).
//   * A TMA warp streams the [256 rows x 128 bytes] code tile (128B-swizzled)
//     and the four [16 x 64] activation boxes of each step into a 3-deep ring.
//   * Sixteen warps own 16 weight rows each.  For every 64-column block they read
//     the rows' 32 code bytes, turn each byte into the two bf16 levels it
//     encodes with one shared-memory load from a 256-entry pair table (one copy
//     per lane: conflict-free), and feed them straight from registers to warp
//     MMAs (m16n8k16, bf16 in, fp32 out): a code byte is exactly one A-fragment
//     register.  The block's product is scaled by its constant
//     c1' = fma(e4m3(q), c2/448, mu) and added to fp32 registers.
//   * The tensor core here only replaces FMAs: per weight it does 2 M FLOP.
//     Warp MMAs are used because a skinny-N product issued as tcgen05.mma
//     from one thread costs about 80 cycles per 128x16x16 instruction, which
//     caps a 16-token stream near 25 weights per cycle per SM, while HBM
//     delivers about 46.
//   * The last CTA to finish a tile (counter) adds s (X A^T) B^T and writes Y.
// Numerics: the block constant multiplies the fp32 product of its block, so a
// weight enters as bf16(L[code]) * c1' rather than bf16(L[code] * c1'): the same
// linear map up to the rounding of each weight.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "gemv.h"
#include "nf4_device.cuh"
#include "sm100_ptx.cuh"

namespace qlora {
namespace {

constexpr int kRows = 256;                     // weight rows per tile
constexpr int kComputeWarps = 16;              // 16 rows (one m16 MMA tile) each
constexpr int kProducerWarp = kComputeWarps;
constexpr int kThreads = (kComputeWarps + 1) * 32;
constexpr int kStages = 3;
constexpr int kStepCols = 256;                 // 4 blocks of 64 columns
constexpr int kCodeTile = kRows * 128;         // 256 rows x 128 bytes, 128B-swizzled
constexpr int kXBox = 16 * 128;                // 16 tokens x 64 bf16, 128B-swizzled
constexpr int kXTile = 4 * kXBox;
constexpr int kTable = 256 * 32 * 4;           // byte value x lane -> bf16 pair
constexpr size_t kSmem = 32768 + kTable + kStages * (kCodeTile + kXTile) + 1024;

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
// Bounded barrier among the compute warps, built on an mbarrier (a named
// bar.sync could not give up if a warp had left after a timed-out wait).
__device__ __forceinline__ bool group_sync(uint64_t* bar, uint32_t& phase, uint32_t* err) {
  mbar_arrive(bar);
  const bool ok = mbar_wait(bar, phase, err);
  phase ^= 1u;
  return ok;
}
// Byte t of the word, times 128, in bits 7..14 (rotate right by 8t - 7).
__device__ __forceinline__ uint32_t byte_x128(uint32_t w, uint32_t rot) {
  uint32_t r;
  asm("shf.r.wrap.b32 %0, %1, %1, %2;" : "=r"(r) : "r"(w), "r"(rot));
  return r & 0x7F80u;
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// CTA i owns global steps [bound(i), bound(i + 1)) of all tiles, tile-major.
__device__ __forceinline__ int64_t bound(int i, int64_t total, int ctas) {
  return (static_cast<int64_t>(i) * total) / ctas;
}
__device__ __forceinline__ int cta_of(int64_t x, int64_t total, int ctas) {
  int i = static_cast<int>((x * ctas) / total);
  while (i + 1 < ctas && bound(i + 1, total, ctas) <= x) ++i;
  while (i > 0 && bound(i, total, ctas) > x) --i;
  return i;
}

template <int kNT>   // n8 token tiles: 1 for M <= 8, 2 for M <= 16
__global__ void __launch_bounds__(kThreads, 1)
k_gemv(const GemvArgs a, const __grid_constant__ CUtensorMap cmap,
       const __grid_constant__ CUtensorMap xmap) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ float s_level[16];
  __shared__ float s_xa[16 * 256];
  __shared__ int s_last;

  const uint32_t raw0 = smem_u32(smem_raw);
  const uint32_t tbl = (raw0 + 32767u) & ~32767u;             // 32 KB aligned pair table
  const uint32_t cs0 = tbl + kTable;                           // code tiles (1024-aligned)
  const uint32_t xs0 = cs0 + kStages * kCodeTile;              // activation tiles
  uint8_t* gen = smem_raw + (tbl - raw0);
  uint64_t* bars = reinterpret_cast<uint64_t*>(gen + kTable + kStages * (kCodeTile + kXTile));
  uint64_t* full = bars;                  // codes + X landed (TMA)
  uint64_t* empty = bars + kStages;       // one arrival per compute warp
  uint64_t* gbar = bars + 2 * kStages;    // compute-warp barrier (all 256 threads)

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t steps = a.steps;
  const int64_t total = static_cast<int64_t>(a.m_tiles) * steps;
  const int64_t x_beg = bound(blockIdx.x, total, gridDim.x);
  const int64_t x_end = bound(blockIdx.x + 1, total, gridDim.x);
  const int kblocks = static_cast<int>(a.kw / 64);

  if (threadIdx.x < 16) s_level[threadIdx.x] = a.level[threadIdx.x];
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kComputeWarps);
    }
    mbar_init(gbar, kComputeWarps * 32);
    fence_barrier_init();
  }
  __syncthreads();
  // pair table: entry (byte b, lane l) = {bf16(L[b >> 4]), bf16(L[b & 15])}, element order
  for (int i = threadIdx.x; i < 256 * 32; i += kThreads) {
    const int b = i >> 5, l = i & 31;
    const __nv_bfloat162 v = __floats2bfloat162_rn(s_level[b >> 4], s_level[b & 15]);
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(tbl + b * 128 + l * 4),
                 "r"(*reinterpret_cast<const uint32_t*>(&v)) : "memory");
  }
  __syncthreads();

  if (warp == kProducerWarp) {
    if (lane == 0) {
      for (int64_t x = x_beg; x < x_end; ++x) {
        const uint32_t it = static_cast<uint32_t>(x - x_beg);
        const uint32_t s = it % kStages, ph = (it / kStages) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, a.err)) break;
        const int tile = static_cast<int>(x / steps);
        const int col0 = static_cast<int>(x % steps) * kStepCols;
        mbar_arrive_expect_tx(&full[s], kCodeTile + kXTile);
        tma_load_2d(gen + kTable + s * kCodeTile, &cmap, col0 / 2, tile * kRows, &full[s]);
#pragma unroll
        for (int b = 0; b < 4; ++b)
          tma_load_2d(gen + kTable + kStages * kCodeTile + s * kXTile + b * kXBox, &xmap, col0 + b * 64, 0,
                      &full[s]);
      }
    }
    return;
  }

  // ------------------------------------------------ compute warps
  const int g = lane >> 2, t = lane & 3;
  const uint32_t tlane = tbl + lane * 4;
  const uint32_t rot = (8u * t + 25u) & 31u;                   // 8t - 7 mod 32
  const float mu = __ldg(a.mean);
  float y[kNT][4];
#pragma unroll
  for (int n = 0; n < kNT; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) y[n][e] = 0.0f;

  // Block-constant inputs (E4M3 byte, c2) of lane t's block in the warp's two
  // rows, loaded two steps before their use (two register slots, alternating).
  // qv[r] packs the E4M3 byte (bits 0..7) and the c2 group index (bits 8..);
  // a row's group changes only every 256 blocks, so c2 / 448 is cached below.
  auto load_raw = [&](int64_t xx, uint32_t (&qv)[2], float (&cv)[2]) {
    const int tl = static_cast<int>(xx / steps);
    const int kb = static_cast<int>(xx % steps) * 4 + t;
    const int64_t r0 = static_cast<int64_t>(tl) * kRows + warp * 16 + g;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int64_t n = r0 + 8 * r;
      qv[r] = 0xFFFFFFFFu;                         // marks "no block": constant 0
      cv[r] = 0.0f;
      if (xx < x_end && n < a.nw && kb < kblocks) {
        const int64_t blk = n * kblocks + kb;
        qv[r] = __ldg(a.qabs + blk) | (static_cast<uint32_t>(blk >> 8) << 8);
        cv[r] = __ldg(a.c2 + (blk >> 8));
      }
    }
  };
  uint32_t grp_cache[2] = {0xFFFFFFFFu, 0xFFFFFFFFu};
  float c2q_cache[2] = {0.0f, 0.0f};

  bool alive = true;
  uint32_t gphase = 0;
  // One step: wait for its stage, decode + multiply its four blocks, release
  // the stage, and at the end of this CTA's share of a tile add the partial.
  auto process = [&](int64_t x, uint32_t (&qv)[2], float (&cv)[2]) {
    const uint32_t it = static_cast<uint32_t>(x - x_beg);
    const uint32_t s = it % kStages, ph = (it / kStages) & 1u;
    const int tile = static_cast<int>(x / steps);
    const int step = static_cast<int>(x % steps);
    const int64_t row0 = static_cast<int64_t>(tile) * kRows + warp * 16 + g;   // rows row0, row0 + 8
    float cmine[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      cmine[r] = 0.0f;
      if (qv[r] != 0xFFFFFFFFu) {
        const uint32_t grp = qv[r] >> 8;
        if (grp != grp_cache[r]) {
          grp_cache[r] = grp;
          c2q_cache[r] = __fdiv_rn(cv[r], 448.0f);
        }
        cmine[r] = block_constant(qv[r] & 0xFFu, c2q_cache[r], mu);
      }
    }
    load_raw(x + 2, qv, cv);
    if (!mbar_wait(&full[s], ph, a.err)) { alive = false; return; }
    const uint32_t cs = cs0 + s * kCodeTile + (warp * 16 + g) * 128;
    const uint32_t xs = xs0 + s * kXTile;
#pragma unroll 2
    for (int b = 0; b < 4; ++b) {
      // code words of the two rows for block b (logical chunks 2b, 2b+1; swizzle key g)
      uint32_t w[2][8];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const uint32_t rb = cs + r * 8 * 128;
        const uint4 lo = lds128(rb + (((2 * b) ^ g) << 4));
        const uint4 hi = lds128(rb + (((2 * b + 1) ^ g) << 4));
        w[r][0] = lo.x; w[r][1] = lo.y; w[r][2] = lo.z; w[r][3] = lo.w;
        w[r][4] = hi.x; w[r][5] = hi.y; w[r][6] = hi.z; w[r][7] = hi.w;
      }
      float p[2][kNT][4];                           // two chains: even / odd slices
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int n = 0; n < kNT; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) p[c][n][e] = 0.0f;
      const uint32_t xb = xs + b * kXBox;
#pragma unroll
      for (int j = 0; j < 4; ++j) {               // 16-column slices of the block
        uint32_t bf[kNT][2];
#pragma unroll
        for (int n = 0; n < kNT; ++n) {
          const uint32_t xr = xb + (8 * n + g) * 128 + 4 * t;
          bf[n][0] = lds32(xr + (((2 * j) ^ g) << 4));
          bf[n][1] = lds32(xr + (((2 * j + 1) ^ g) << 4));
        }
        const uint32_t a0 = lds32(tlane | byte_x128(w[0][2 * j], rot));
        const uint32_t a1 = lds32(tlane | byte_x128(w[1][2 * j], rot));
        const uint32_t a2 = lds32(tlane | byte_x128(w[0][2 * j + 1], rot));
        const uint32_t a3 = lds32(tlane | byte_x128(w[1][2 * j + 1], rot));
#pragma unroll
        for (int n = 0; n < kNT; ++n) mma_bf16_16816(p[j & 1][n], a0, a1, a2, a3, bf[n][0], bf[n][1]);
      }
      // scale the block's partial by its constants (rows g and g+8)
      const float c_lo = __shfl_sync(0xFFFFFFFFu, cmine[0], (lane & ~3) | b);
      const float c_hi = __shfl_sync(0xFFFFFFFFu, cmine[1], (lane & ~3) | b);
#pragma unroll
      for (int n = 0; n < kNT; ++n) {
        y[n][0] = __fmaf_rn(c_lo, p[0][n][0] + p[1][n][0], y[n][0]);
        y[n][1] = __fmaf_rn(c_lo, p[0][n][1] + p[1][n][1], y[n][1]);
        y[n][2] = __fmaf_rn(c_hi, p[0][n][2] + p[1][n][2], y[n][2]);
        y[n][3] = __fmaf_rn(c_hi, p[0][n][3] + p[1][n][3], y[n][3]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);

    if (step == steps - 1 || x == x_end - 1) {
      // end of this CTA's share of the tile: add the partial, maybe finish the tile
#pragma unroll
      for (int n = 0; n < kNT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int64_t row = row0 + 8 * (e >> 1);
          const int tok = 8 * n + 2 * t + (e & 1);
          if (row < a.nw && tok < a.m) atomicAdd(a.yacc + tok * a.nw + row, y[n][e]);
          y[n][e] = 0.0f;
        }
      __threadfence();
      if (!group_sync(gbar, gphase, a.err)) { alive = false; return; }
      if (threadIdx.x == 0) {
        const int first = cta_of(static_cast<int64_t>(tile) * steps, total, gridDim.x);
        const int last = cta_of(static_cast<int64_t>(tile + 1) * steps - 1, total, gridDim.x);
        s_last = (atomicAdd(a.counters + tile, 1) == last - first) ? 1 : 0;
      }
      if (!group_sync(gbar, gphase, a.err)) { alive = false; return; }
      if (s_last) {
        __threadfence();
        for (int e = threadIdx.x; e < a.m * a.r; e += kComputeWarps * 32)
          s_xa[e] = __ldcg(a.xa + (e / a.r) * a.ld_xa + (e % a.r));
        if (!group_sync(gbar, gphase, a.err)) { alive = false; return; }
        const int64_t n = static_cast<int64_t>(tile) * kRows + threadIdx.x;
        if (threadIdx.x < kRows && n < a.nw) {
          float lo[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) lo[i] = 0.0f;
          const uint4* brow = reinterpret_cast<const uint4*>(a.lora_b + n * a.r);
          for (int c = 0; c < a.r / 8; ++c) {
            const uint4 bv = __ldg(brow + c);
            const float b8[8] = {bf16_lo(bv.x), bf16_hi(bv.x), bf16_lo(bv.y), bf16_hi(bv.y),
                                 bf16_lo(bv.z), bf16_hi(bv.z), bf16_lo(bv.w), bf16_hi(bv.w)};
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (i < a.m) {
#pragma unroll
                for (int e = 0; e < 8; ++e) lo[i] = __fmaf_rn(s_xa[i * a.r + c * 8 + e], b8[e], lo[i]);
              }
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if (i < a.m) {
              const float acc = __ldcg(a.yacc + i * a.nw + n);
              const __nv_bfloat16 v = __float2bfloat16_rn(__fmaf_rn(a.s, lo[i], acc));
              a.y[i * a.nw + n] = *reinterpret_cast<const uint16_t*>(&v);
            }
          }
        }
        if (!group_sync(gbar, gphase, a.err)) { alive = false; return; }
      }
    }
  };

  uint32_t qa[2], qb[2];
  float ca[2], cb[2];
  load_raw(x_beg, qa, ca);
  load_raw(x_beg + 1, qb, cb);
  for (int64_t x = x_beg; x < x_end && alive; x += 2) {
    process(x, qa, ca);
    if (x + 1 < x_end && alive) process(x + 1, qb, cb);
  }
}

// X A^T for M <= 16 tokens: block j reduces column j over all of K in fp32.
// Also zeroes k_gemv's split buffer and tile counters (grid-stride).
__global__ void __launch_bounds__(256)
k_xa_small(const uint16_t* __restrict__ X, const uint16_t* __restrict__ A, int64_t m, int64_t kw, int r,
           float* __restrict__ xa, int64_t ld, float* __restrict__ xa_out, float* __restrict__ zero_f,
           int64_t zero_n, int* __restrict__ zero_i, int zero_ni) {
  __shared__ float s_red[8][16];
  const int j = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
  const int64_t nchunks = kw / 8;
  for (int64_t c = threadIdx.x; c < nchunks; c += blockDim.x) {
    const uint4 av = __ldg(reinterpret_cast<const uint4*>(A + j * kw) + c);
    const float af[8] = {bf16_lo(av.x), bf16_hi(av.x), bf16_lo(av.y), bf16_hi(av.y),
                         bf16_lo(av.z), bf16_hi(av.z), bf16_lo(av.w), bf16_hi(av.w)};
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (i < m) {
        const uint4 xv = __ldg(reinterpret_cast<const uint4*>(X + i * kw) + c);
        const float xf[8] = {bf16_lo(xv.x), bf16_hi(xv.x), bf16_lo(xv.y), bf16_hi(xv.y),
                             bf16_lo(xv.z), bf16_hi(xv.z), bf16_lo(xv.w), bf16_hi(xv.w)};
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[i] = __fmaf_rn(af[e], xf[e], acc[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc[i] += __shfl_xor_sync(0xFFFFFFFFu, acc[i], o);
  }
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < 16; ++i) s_red[warp][i] = acc[i];
  }
  __syncthreads();
  if (threadIdx.x < m) {
    float v = 0.0f;
    for (int w = 0; w < 8; ++w) v += s_red[w][threadIdx.x];
    xa[threadIdx.x * ld + j] = v;
    if (xa_out) xa_out[threadIdx.x * r + j] = v;
  }
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (int64_t i = gtid; i < zero_n; i += nthreads) zero_f[i] = 0.0f;
  for (int64_t i = gtid; i < zero_ni; i += nthreads) zero_i[i] = 0;
}

template <int kNT>
cudaError_t launch_gemv_t(const GemvArgs& args, const CUtensorMap& cm, const CUtensorMap& xm, int num_sms,
                          cudaStream_t stream) {
  static std::atomic<uint64_t> attr_done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_done.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(k_gemv<kNT>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmem));
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(bit, std::memory_order_acq_rel);
  }
  const int64_t total = static_cast<int64_t>(args.m_tiles) * args.steps;
  const int grid = static_cast<int>(total < num_sms ? total : num_sms);
  k_gemv<kNT><<<grid, kThreads, kSmem, stream>>>(args, cm, xm);
  return cudaGetLastError();
}

}  // namespace

int gemv_tile_rows() { return kRows; }

cudaError_t launch_xa_small(const uint16_t* X, const uint16_t* A, int64_t m, int64_t kw, int r, float* xa,
                            int64_t ld, float* xa_out, float* zero_f, int64_t zero_n, int* zero_i,
                            int zero_ni, cudaStream_t stream) {
  k_xa_small<<<r, 256, 0, stream>>>(X, A, m, kw, r, xa, ld, xa_out, zero_f, zero_n, zero_i, zero_ni);
  return cudaGetLastError();
}

cudaError_t launch_gemv(const GemvArgs& args, const CUtensorMap& codes_map, const CUtensorMap& x_map,
                        int num_sms, cudaStream_t stream) {
  if (args.m <= 8) return launch_gemv_t<1>(args, codes_map, x_map, num_sms, stream);
  return launch_gemv_t<2>(args, codes_map, x_map, num_sms, stream);
}

}  // namespace qlora
