// gemv.cu -- decode-shaped forward of the NF4 LoRA linear layer (M <= 16 tokens).
//
// Y = X deq(W)^T + s (X A^T) B^T with few token rows is a stream over the packed
// weight (automatone "QLoRA paper explained", section "How it works": the 4-bit
// weight is dequantized on the fly for the matmul), bound by HBM.  Two kernels,
// the second launched as the programmatic dependent of the first:
//
// k_xa_zero: partial X A^T over slices of K in fp32 (CUDA cores), and the
//   zeroed tile counters of k_gemv.
//
// k_gemv: the weight stream and the whole output.  Each CTA takes an equal,
//   contiguous share of all (256-row tile, 256-column step) pairs, so the work
//   is balanced whatever the shape.
//   * Four producer warps, one per SM sub-partition: one lane streams the
//     [256 rows x 128 bytes] code tile (128B-swizzled) and the four [m x 64]
//     activation boxes of each step into a 3- or 4-deep ring (TMA), and the
//     warps write the step's block constants c1' = fma(e4m3(q), c2/448, mu)
//     (or, for a weight stored without double quantization, its fp32 c1)
//     into the stage.
//   * Eight consumer warps own 32 weight rows each.  For every 64-column block
//     they read their rows' code bytes, turn each byte into the two bf16 levels
//     it encodes with one shared-memory load from a 256-entry pair table (one
//     copy per lane: conflict-free), and feed them straight from registers to
//     warp MMAs (m16n8k16, bf16 in, fp32 out): a code byte is exactly one
//     A-fragment register.  The block's product is scaled by its constant and
//     added to fp32 registers.
//   * A tile that lies in one CTA's share is finished by that CTA at once.
//     For a shared tile each warp writes its fp32 partial to one of its CTA's
//     two slots; the warp whose partial completes the tile's 32 rows (a
//     per-warp counter) sums the slots of the tile's CTAs, adds the LoRA
//     up-projection with warp MMAs over the staged bf16(s X A^T) and writes
//     those rows of Y.  At the end of its share a warp that finds every other
//     part already counted finishes without writing or counting its own.
//   * The producer warpgroup gives registers to the consumers after the start
//     (setmaxnreg), so that the consumers' loop runs without spills.
//   * The tensor core here only replaces FMAs: per weight it does 2 M FLOP.
//     Warp MMAs are used because a skinny-N product issued as tcgen05.mma
//     from one thread costs about 80 cycles per 128x16x16 instruction, which
//     caps a 16-token stream near 25 weights per cycle per SM, while HBM
//     delivers about 46.
//
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
constexpr int kStepCols = 256;                 // 4 blocks of 64 columns
constexpr uint32_t kCodeTile = kRows * 128;    // 256 rows x 128 bytes, 128B-swizzled
// Shared-memory map (addresses in the CTA's shared window).  The pair table
// sits at a 64 KB boundary so that one byte-permute builds a lookup address:
// entry (code byte v, lane l) lives at kTableAddr + v * 256 + l * 4.  The other
// half of each 256-byte row holds the block-constant slots, X A^T staging and
// partial.  Below the table: the X stages and code stage 0; above it: code
// stages 1 .. kStages - 1.
constexpr uint32_t kTableAddr = 0x10000;
constexpr uint32_t kHighAddr = 0x20000;
constexpr uint32_t kMiscBytes = 256;           // barriers, levels
// Pipeline depth and X box stride by token tiles: four stages when the X boxes
// (m <= 8 rows of 128 bytes) fit in 1 KB each, three otherwise.
template <int kNT>
struct GemvStages {
  static constexpr int kStages = kNT == 1 ? 4 : 3;
  static constexpr uint32_t kXBox = kNT == 1 ? 1024 : 2048;   // 1 KB aligned (128B swizzle)
  static constexpr uint32_t kXTile = 4 * kXBox;
  static constexpr uint32_t kSmemTop = kHighAddr + (kStages - 1) * kCodeTile;
};

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
// Predicated 16-byte load: when `pred` is false the registers are left as they
// are (their contents are then unspecified and must not matter).
__device__ __forceinline__ uint4 lds128_if(bool pred, uint32_t addr) {
  uint4 v;
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
               "@p ld.shared.v4.b32 {%0, %1, %2, %3}, [%5];\n\t}"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(static_cast<uint32_t>(pred)), "r"(addr));
  return v;
}
// Pair-table read: the table does not change after set-up, so the load may be
// scheduled freely (no volatile).
__device__ __forceinline__ uint32_t lds_table(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}
__device__ __forceinline__ float4 lds128f(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr) : "memory");
  return v;
}
// Free half of pair-table row `row` (128 bytes at kTableAddr + row * 256 + 128).
__device__ __forceinline__ uint32_t hole(uint32_t row, uint32_t byte) {
  return kTableAddr + row * 256u + 128u + byte;
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// Same with a zero accumulator input (the first product of a chain).
__device__ __forceinline__ void mma_bf16_16816_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                                 uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %10, %10, %10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}
// Four E4M3 bytes -> floats (exact: every E4M3 value is a normal f16 or zero).
__device__ __forceinline__ void e4m3x4_to_f32(uint32_t q, float (&f)[4]) {
  uint32_t lo, hi;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi) : "r"(q));
  f[0] = __half2float(__ushort_as_half(static_cast<unsigned short>(lo & 0xFFFFu)));
  f[1] = __half2float(__ushort_as_half(static_cast<unsigned short>(lo >> 16)));
  f[2] = __half2float(__ushort_as_half(static_cast<unsigned short>(hi & 0xFFFFu)));
  f[3] = __half2float(__ushort_as_half(static_cast<unsigned short>(hi >> 16)));
}
// Named barriers: 1 between the producer warps (arrive, do not wait) and the
// consumer warps (wait for all `count` threads); 2 among the producer warps.
__device__ __forceinline__ void named_barrier_arrive(int id, int count) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void named_barrier_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t atomic_add_acq_rel(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;");
}

// CTA i owns global steps [bound(i), bound(i + 1)) of all tiles, tile-major.
__device__ __forceinline__ int64_t bound(int i, int64_t total, int ctas) {
  return (static_cast<int64_t>(i) * total) / ctas;
}
// The CTA whose share holds global step u (ctas <= total, so no share is empty).
__device__ __forceinline__ int64_t owner_of(int64_t u, int64_t total, int ctas) {
  return ((u + 1) * ctas - 1) / total;
}

// Block-constant inputs of one step for one weight row, loaded ahead.  With
// double quantization: the E4M3 bytes of the step's four blocks (byte b =
// block b) in q, and in v[0] c2 of the first block's group (in v[1], when K is
// not a multiple of 256 columns, that of the last block's group too).
// Without it: the four blocks' fp32 constants in v[0..3].
struct RowConsts {
  uint32_t q;
  float v[4];
};

// Eight consumer warps own 32 weight rows each (two m16 MMA tiles); warps
// 8..11 are producers, one per SM sub-partition, so that their work weighs on
// all four schedulers alike.  Each sub-partition then holds three warps:
// 3 x 32 x 168 registers fit its 16K.
constexpr int kConsumerWarps = 8;
constexpr int kProducerWarps = 4;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kGemvThreads = kConsumers + kProducerWarps * 32;
constexpr int kGemvMaxRegs = 168;
// After the start the producer warpgroup hands registers to the consumers:
// 128 x 80 + 256 x 208 = 63,488 of the 384 x 168 = 64,512 the CTA is launched
// with (per SM sub-partition: 2 x 32 x 208 + 32 x 80 = 15,872 <= 3 x 32 x 168).
constexpr int kProducerRegs = 80;
constexpr int kConsumerRegs = 208;
static_assert(kProducerWarps * 32 * kProducerRegs + kConsumers * kConsumerRegs <= kGemvThreads * kGemvMaxRegs,
              "register split exceeds the launch allocation");
constexpr int kRowsPerProducerLane = kRows / (kProducerWarps * 32);
constexpr uint32_t kSxaHole = 128;     // first pair-table hole row of the s X A^T staging
// A CTA that ends its part of its first tile within this many steps of its
// start counts that part at its next tile end instead (the previous kernel,
// which zeroes the counters, may still be running that early).
constexpr int64_t kDeferSteps = 3;

template <int kNT, bool kQuad>   // kNT: n8 token tiles (1: M <= 8, 2: M <= 16); kQuad: K % 256 == 0
__global__ void __maxnreg__(kGemvMaxRegs)
k_gemv(const GemvArgs a, const __grid_constant__ CUtensorMap cmap,
       const __grid_constant__ CUtensorMap xmap) {
  constexpr int kStages = GemvStages<kNT>::kStages;
  constexpr uint32_t kXBox = GemvStages<kNT>::kXBox;
  constexpr uint32_t kXTile = GemvStages<kNT>::kXTile;
  constexpr uint32_t kSmemTop = GemvStages<kNT>::kSmemTop;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw0 = smem_u32(smem_raw);
  uint32_t dyn_bytes;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_bytes));
  const uint32_t xs0 = (raw0 + 1023u) & ~1023u;              // X stages (4 boxes each)
  const uint32_t cs_low = xs0 + kStages * kXTile;            // code stage 0
  const uint32_t misc = cs_low + kCodeTile;
  if (misc + kMiscBytes > kTableAddr || raw0 + dyn_bytes < kSmemTop) {
    if (threadIdx.x == 0) atomicOr(a.err, kErrSmemLayout);
    return;
  }
  auto gptr = [&](uint32_t addr) { return smem_raw + (addr - raw0); };
  auto code_stage = [&](uint32_t s) { return s == 0 ? cs_low : kHighAddr + (s - 1) * kCodeTile; };
  uint64_t* bars = reinterpret_cast<uint64_t*>(gptr(misc));
  uint64_t* full = bars;                  // codes + X landed (TMA) and constants written (producer)
  uint64_t* empty = bars + kStages;       // one arrival per consumer warp
  uint64_t* xa_bar = bars + 2 * kStages;  // s X A^T staged (one arrival per consumer warp)

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t steps = a.steps;
  const int64_t total = static_cast<int64_t>(a.m_tiles) * steps;
  const int ctas = static_cast<int>(gridDim.x);
  const int64_t x_beg = bound(blockIdx.x, total, ctas);
  const int64_t x_end = bound(blockIdx.x + 1, total, ctas);
  const int kblocks = static_cast<int>(a.kw / 64);
  const uint32_t kbl = static_cast<uint32_t>(kblocks);
  const int m = static_cast<int>(a.m);

  // Position of a step: (tile, step within the tile's row of steps).  Advanced
  // incrementally so that no 64-bit division runs per step.
  struct Pos {
    int tile, step;
  };
  auto advance = [&](Pos p) {
    if (++p.step == steps) { p.step = 0; ++p.tile; }
    return p;
  };
  const int64_t n_mine = x_end - x_beg;
  const Pos first{static_cast<int>(x_beg / steps), static_cast<int>(x_beg % steps)};

  // Block constants of step p for tile rows lane + 32 j (j < 8), staged in the
  // free halves of the pair-table rows: slot s holds row r's four constants at
  // hole(32 s + r / 8, 16 (r mod 8)).
  const uint32_t xbytes = 4u * static_cast<uint32_t>(m) * 128u;
  // the loads of one stage: the code tile and the four activation boxes of step p
  auto issue_stage = [&](Pos p, uint32_t st) {
    mbar_arrive_expect_tx(&full[st], kCodeTile + xbytes);
    const int col0 = p.step * kStepCols;
    tma_load_2d(gptr(code_stage(st)), &cmap, col0 / 2, p.tile * kRows, &full[st]);
#pragma unroll
    for (int b = 0; b < 4; ++b)
      tma_load_2d(gptr(xs0 + st * kXTile + b * kXBox), &xmap, col0 + b * 64, 0, &full[st]);
  };
  if (threadIdx.x == kConsumers) {
    tma_prefetch_desc(&cmap);
    tma_prefetch_desc(&xmap);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1 + kProducerWarps);
      mbar_init(&empty[i], kConsumerWarps);
    }
    mbar_init(xa_bar, kConsumerWarps);
    fence_barrier_init();
  }
  if (warp >= kConsumerWarps) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
    // ------------------------------------------------ producer warps
    // Thread 0 of warp 8 streams the [256 rows x 128 bytes] code tile
    // (128B-swizzled) and the four [m x 64] activation boxes of each step into
    // the ring; producer warp h writes the step's block constants of tile rows
    // 64 h + lane + 32 j (j < 2) into the stage's slot.  The consumers only wait
    // for the barrier initialisation.
    const int hw = warp - kConsumerWarps;
    const bool tma_thread = hw == 0 && lane == 0;
    named_barrier_sync(2, kProducerWarps * 32);   // barrier initialisation seen by all producers
    named_barrier_arrive(1, kGemvThreads);
    const float mu = a.absf != nullptr ? 0.0f : __ldg(a.mean);
    const bool plain = a.absf != nullptr;
    auto load_raw = [&](Pos p, bool valid, RowConsts (&k)[kRowsPerProducerLane]) {
#pragma unroll
      for (int j = 0; j < kRowsPerProducerLane; ++j) {
        k[j].q = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) k[j].v[b] = 0.0f;
        const int64_t row = static_cast<int64_t>(p.tile) * kRows + 64 * hw + lane + 32 * j;
        if (valid && row < a.nw) {
          const uint32_t blk0 = static_cast<uint32_t>(row) * kbl + 4u * static_cast<uint32_t>(p.step);
          if (plain) {
            if (kQuad) {           // blk0 is a multiple of 4: one 16-byte load
              const float4 f = __ldg(reinterpret_cast<const float4*>(a.absf + blk0));
              k[j].v[0] = f.x; k[j].v[1] = f.y; k[j].v[2] = f.z; k[j].v[3] = f.w;
            } else {
              const int nb = min(4, kblocks - 4 * p.step);
#pragma unroll
              for (int b = 0; b < 4; ++b)
                if (b < nb) k[j].v[b] = __ldg(a.absf + blk0 + b);
            }
          } else if (kQuad) {
            k[j].q = __ldg(reinterpret_cast<const uint32_t*>(a.qabs + blk0));
            k[j].v[0] = __ldg(a.c2 + (blk0 >> 8));
          } else {
            const int nb = min(4, kblocks - 4 * p.step);
#pragma unroll
            for (int b = 0; b < 4; ++b)
              if (b < nb) k[j].q |= static_cast<uint32_t>(__ldg(a.qabs + blk0 + b)) << (8 * b);
            k[j].v[0] = __ldg(a.c2 + (blk0 >> 8));
            k[j].v[1] = __ldg(a.c2 + ((blk0 + nb - 1) >> 8));
          }
        }
      }
    };
    // c2 / 448 of the group last seen by each of the lane's rows
    uint32_t grp_cache[kRowsPerProducerLane];
    float c2q_cache[kRowsPerProducerLane];
#pragma unroll
    for (int j = 0; j < kRowsPerProducerLane; ++j) { grp_cache[j] = 0xFFFFFFFFu; c2q_cache[j] = 0.0f; }
    // c[b] = fma(e4m3(q_b), c2 / 448, mu) for the lane's rows of step p into slot `slot`
    auto write_consts = [&](Pos p, const RowConsts (&k)[kRowsPerProducerLane], uint32_t slot) {
#pragma unroll
      for (int j = 0; j < kRowsPerProducerLane; ++j) {
        const int64_t row = static_cast<int64_t>(p.tile) * kRows + 64 * hw + lane + 32 * j;
        const uint32_t blk0 = static_cast<uint32_t>(row) * kbl + 4u * static_cast<uint32_t>(p.step);
        const uint32_t grp = blk0 >> 8;
        float c[4];
        if (plain) {
#pragma unroll
          for (int b = 0; b < 4; ++b) c[b] = k[j].v[b];
        } else {
          if (grp != grp_cache[j]) {
            grp_cache[j] = grp;
            c2q_cache[j] = __fdiv_rn(k[j].v[0], 448.0f);
          }
          float f[4];
          e4m3x4_to_f32(k[j].q, f);
          if (kQuad) {
#pragma unroll
            for (int b = 0; b < 4; ++b) c[b] = __fmaf_rn(f[b], c2q_cache[j], mu);
          } else {
            const float c2q_b = __fdiv_rn(k[j].v[1], 448.0f);
#pragma unroll
            for (int b = 0; b < 4; ++b)
              c[b] = __fmaf_rn(f[b], ((blk0 + b) >> 8) == grp ? c2q_cache[j] : c2q_b, mu);
          }
        }
        const uint32_t r = static_cast<uint32_t>(64 * hw + lane + 32 * j);
        sts128(hole(32u * slot + (r >> 3), (r & 7u) * 16u), c[0], c[1], c[2], c[3]);
      }
    };
    Pos p = first;
    Pos p2 = advance(advance(first));
    RowConsts ra[kRowsPerProducerLane], rb[kRowsPerProducerLane];                // raw constants of steps it and it + 1
    load_raw(first, n_mine > 0, ra);
    load_raw(advance(first), n_mine > 1, rb);
    uint32_t ps = 0, pph = 0;
    for (int64_t it = 0; it < n_mine; ++it) {
      RowConsts rc[kRowsPerProducerLane];
      load_raw(p2, it + 2 < n_mine, rc);  // two steps ahead
      // stage ps is free once every consumer warp released its previous use
      bool ok = true;
      if (lane == 0) ok = mbar_test_wait(&empty[ps], pph ^ 1u) || mbar_wait(&empty[ps], pph ^ 1u, a.err);
      if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) break;
      if (tma_thread) issue_stage(p, ps);
      write_consts(p, ra, ps);
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[ps]);   // the warp's constant stores are ordered before it
#pragma unroll
      for (int j = 0; j < kRowsPerProducerLane; ++j) { ra[j] = rb[j]; rb[j] = rc[j]; }
      p = advance(p);
      p2 = advance(p2);
      if (++ps == kStages) { ps = 0; pph ^= 1u; }
    }
    return;
  }
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kConsumerRegs));
  // pair table: entry (byte v, lane l) = {bf16(L[v >> 4]), bf16(L[v & 15])}, element order;
  // consumer thread v converts entry v once and writes its 32 copies
  {
    const int v = threadIdx.x;
    const __nv_bfloat162 e = __floats2bfloat162_rn(a.level[v >> 4], a.level[v & 15]);
    const float ev = __uint_as_float(*reinterpret_cast<const uint32_t*>(&e));
#pragma unroll
    for (int l = 0; l < 32; l += 4) sts128(kTableAddr + v * 256 + l * 4, ev, ev, ev, ev);
  }
  named_barrier_sync(1, kGemvThreads);    // pair table written, barriers initialised

  // ------------------------------------------------ consumer warps
  // Lane (g, t) serves MMA rows g and g + 8 of the warp's two m16 tiles.  MMA
  // row g of an 8-row group is weight row 8u + pg with pg = 2(g mod 4) + g / 4,
  // so that the lanes of each half-warp read rows whose 128-byte swizzle
  // patterns differ in bits 1 and 2 (no bank conflicts).  The lane's rows are
  // warp*32 + 8q + pg (q < 4; tile i uses q = 2i and 2i + 1).  In every
  // 64-column block the lane reads the code bytes [8t, 8t + 8) of those rows.
  // Columns enter the MMA in a permuted order (the same for X): slice j of a
  // block feeds columns 16t + 4j + {0, 1} as k = {2t, 2t+1} and 16t + 4j + {2, 3}
  // as k = {2t+8, 2t+9}, so every lane reads only its own bytes.  The LoRA
  // up-projection uses the same order over each 64-column group of the rank.
  const int g = lane >> 2, t = lane & 3;
  const int pg = ((g & 3) << 1) | (g >> 2);
  const uint32_t tbase = kTableAddr | (static_cast<uint32_t>(lane) << 2);
  const uint32_t crow = static_cast<uint32_t>(warp * 32 + pg) * 128u;

  // X rows of this lane (token 8n + g); lanes of tokens >= m load nothing, and
  // the MMA columns they feed are never stored.
  bool xon[kNT];
  uint32_t xoff[kNT][2];
#pragma unroll
  for (int n = 0; n < kNT; ++n) {
    xon[n] = 8 * n + g < m;
#pragma unroll
    for (int jp = 0; jp < 2; ++jp) xoff[n][jp] = (8 * n + g) * 128 + ((((2u * t) + jp) ^ g) << 4);
  }

  // s X A^T as bf16 [token][64 lora_steps]: 16-byte chunk c of token i's
  // 64-column group q sits in hole row kSxaHole + i lora_steps + q at chunk
  // c ^ (i mod 8), so that the eight tokens read by a quarter-warp hit
  // different banks.
  auto sxa_addr = [&](int tok, int grp, int chunk) -> uint32_t {
    return hole(kSxaHole + static_cast<uint32_t>(tok * a.lora_steps + grp),
                static_cast<uint32_t>((chunk ^ (tok & 7)) << 4));
  };
  // Sum k_xa_zero's K slices of X A^T, write X A^T out from CTA 0 when asked,
  // and stage bf16(s X A^T).  One lane per (8-column chunk, slice): the slices
  // of a chunk sit in 2^sb adjacent lanes and are added by a butterfly of
  // shuffles, so a round costs one load latency whatever the slice count.
  auto stage_sxa = [&]() {
    const int c8n = a.lora_steps * 8;               // 8-column chunks per token
    const int nchunk = m * c8n;
    int sb = 0;
    while ((1 << sb) < a.xa_splits) ++sb;           // at most 4 (16 slices)
    const int sp = static_cast<int>(threadIdx.x) & ((1 << sb) - 1);
    for (int e0 = 0; e0 < nchunk; e0 += kConsumers >> sb) {
      const int e = e0 + (static_cast<int>(threadIdx.x) >> sb);
      const int tok = e / c8n, c8 = e - (e / c8n) * c8n;
      const int col = 8 * c8;
      const bool live = e < nchunk && col < a.r;    // r is a multiple of 8
      float v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = 0.0f;
      if (live && sp < a.xa_splits) {
        const float4* src =
            reinterpret_cast<const float4*>(a.xa_part + (static_cast<int64_t>(sp) * 16 + tok) * a.ld_xa + col);
        const float4 u0 = __ldcg(src), u1 = __ldcg(src + 1);
        v[0] = u0.x; v[1] = u0.y; v[2] = u0.z; v[3] = u0.w;
        v[4] = u1.x; v[5] = u1.y; v[6] = u1.z; v[7] = u1.w;
      }
      for (int o = 1; o < (1 << sb); o <<= 1)
#pragma unroll
        for (int q = 0; q < 8; ++q) v[q] += __shfl_xor_sync(0xFFFFFFFFu, v[q], o);
      if (sp == 0 && e < nchunk) {
        if (live && a.xa_out && blockIdx.x == 0)
#pragma unroll
          for (int q = 0; q < 8; ++q) a.xa_out[static_cast<int64_t>(tok) * a.r + col + q] = v[q];
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(a.s, v[2 * q]), __fmul_rn(a.s, v[2 * q + 1]));
          w[q] = *reinterpret_cast<const uint32_t*>(&h);
        }
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sxa_addr(tok, c8 >> 3, c8 & 7)),
                     "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]) : "memory");
      }
    }
  };
  // Per-token adapters, read once: lane j < m holds token j's adapter (-1 for
  // none or out of range), and bit j of first_use marks the token that uses
  // its adapter first, so the adapters in use are visited in order of first
  // use without reading the index array again.
  int my_ad = -1;
  uint32_t first_use = 1u;                          // one pass for the single adapter
  if (a.adapter_idx != nullptr) {
    if (lane < m) my_ad = __ldg(a.adapter_idx + lane);
    if (my_ad >= a.n_adapters) my_ad = -1;
    const uint32_t same = __match_any_sync(0xFFFFFFFFu, my_ad);
    const bool first = my_ad >= 0 && (same & ((1u << lane) - 1u)) == 0;
    first_use = __ballot_sync(0xFFFFFFFFu, first);
  }
  auto for_each_adapter = [&](auto&& fn) {
    for (uint32_t mk = first_use; mk != 0; mk &= mk - 1u) fn(__shfl_sync(0xFFFFFFFFu, my_ad, __ffs(mk) - 1));
  };
  // The LoRA up-projection s (X A^T) B^T of one adapter added to this lane's
  // fp32 sums with warp MMAs: A operand = rows of that adapter's B (lb), B
  // operand = the staged bf16(s X A^T) of the tokens `use` selects (the other
  // tokens enter as zeros).
  auto lora_pass = [&](int tile, const uint16_t* __restrict__ lb, const bool (&use)[kNT],
                       float (&acc)[2][kNT][4]) {
    const int64_t row0 = static_cast<int64_t>(tile) * kRows + warp * 32 + pg;
    for (int grp = 0; grp < a.lora_steps; ++grp) {
      uint4 xs[kNT][2];
#pragma unroll
      for (int n = 0; n < kNT; ++n)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint4 u;
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w)
                       : "r"(sxa_addr(8 * n + g, grp, 2 * t + hf)) : "memory");
          xs[n][hf] = use[n] ? u : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        uint4 bv[2][2];                             // [row half][8-column half]
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int64_t row = row0 + 8 * (2 * i + h);
            const int col = grp * 64 + 16 * t + 8 * hf;
            bv[h][hf] = (row < a.nw && col < a.r)
                            ? __ldg(reinterpret_cast<const uint4*>(lb + row * a.r + col))
                            : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const uint32_t a0 = kk ? bv[0][hf].z : bv[0][hf].x, a1 = kk ? bv[1][hf].z : bv[1][hf].x;
            const uint32_t a2 = kk ? bv[0][hf].w : bv[0][hf].y, a3 = kk ? bv[1][hf].w : bv[1][hf].y;
#pragma unroll
            for (int n = 0; n < kNT; ++n) {
              const uint32_t b0 = kk ? xs[n][hf].z : xs[n][hf].x, b1 = kk ? xs[n][hf].w : xs[n][hf].y;
              mma_bf16_16816(acc[i][n], a0, a1, a2, a3, b0, b1);
            }
          }
      }
    }
  };
  // Y rows of tile `tile` for this lane from its fp32 sums: add the LoRA term
  // (one pass per adapter in use) and store bf16.
  auto finish = [&](int tile, float (&acc)[2][kNT][4]) {
    const int64_t row0 = static_cast<int64_t>(tile) * kRows + warp * 32 + pg;
    if (a.adapter_idx == nullptr) {
      bool all[kNT];
#pragma unroll
      for (int n = 0; n < kNT; ++n) all[n] = true;
      lora_pass(tile, a.lora_b, all, acc);
    } else {
      for_each_adapter([&](int ad) {
        bool use[kNT];
#pragma unroll
        for (int n = 0; n < kNT; ++n) use[n] = __shfl_sync(0xFFFFFFFFu, my_ad, 8 * n + g) == ad;
        lora_pass(tile, a.lora_b + static_cast<int64_t>(ad) * a.b_stride, use, acc);
      });
    }
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int n = 0; n < kNT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int64_t row = row0 + 8 * (2 * i + (e >> 1));
          const int tok = 8 * n + 2 * t + (e & 1);
          if (row < a.nw && tok < m) {
            const __nv_bfloat16 h = __float2bfloat16_rn(acc[i][n][e]);
            a.y[tok * a.nw + row] = *reinterpret_cast<const uint16_t*>(&h);
          }
        }
  };
  // Tile partials.  A CTA's share touches at most two tiles that other CTAs
  // share too, its first and its last; every tile inside the share lies in
  // it alone and is finished at once.  At the end of its part of a shared
  // tile a warp writes its fp32 partial to one of the CTA's two slots (plain
  // stores, [cta][2][warp][lane][16] floats) and counts itself in the tile's
  // per-warp counter; the warp whose arrival completes the count sums the
  // slots of every CTA of the tile in CTA order and finishes those 32 rows.
  auto shares_of = [&](int tile) -> int {
    const int64_t u0 = static_cast<int64_t>(tile) * steps;
    return static_cast<int>(owner_of(u0 + steps - 1, total, ctas) - owner_of(u0, total, ctas) + 1);
  };
  auto slot_ptr = [&](int64_t cta, int sl) -> float4* {
    return reinterpret_cast<float4*>(a.slots + (((cta * 2 + sl) * kConsumerWarps + warp) * 32 + lane) * 16);
  };
  auto put_slot = [&](int sl, const float (&v)[2][kNT][4]) {
    float4* d = slot_ptr(blockIdx.x, sl);
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int n = 0; n < kNT; ++n) d[i * kNT + n] = make_float4(v[i][n][0], v[i][n][1], v[i][n][2], v[i][n][3]);
  };
  // count this warp's partial of `tile` (already in its slot); the last one
  // finishes the tile, with `v` as scratch
  auto arrive = [&](int tile, float (&v)[2][kNT][4]) {
    const int shares = shares_of(tile);
    // release: the warp's slot stores are ordered before lane 0's count (warp
    // barrier, then a release atomic); acquire: the last warp sees every slot
    // stored before the counts it read
    __syncwarp();
    uint32_t before = 0;
    if (lane == 0) before = atomic_add_acq_rel(a.cnt + static_cast<int64_t>(tile) * kConsumerWarps + warp, 1u);
    before = __shfl_sync(0xFFFFFFFFu, before, 0);
    if (static_cast<int>(before) + 1 != shares) return;
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int n = 0; n < kNT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) v[i][n][e] = 0.0f;
    const int64_t u0 = static_cast<int64_t>(tile) * steps;
    const int64_t c0 = owner_of(u0, total, ctas);
    // slots in CTA order, kBatch of them in flight at a time (one for 16 tokens,
    // whose step loop leaves no registers to spare)
    constexpr int kBatch = kNT == 1 ? 4 : 1;
    for (int k0 = 0; k0 < shares; k0 += kBatch) {
      float4 q[kBatch][2 * kNT];
#pragma unroll
      for (int k = 0; k < kBatch; ++k)
        if (k0 + k < shares) {
          const int64_t c = c0 + k0 + k;
          // the tile is CTA c's first tile unless c's share starts before it
          const float4* src = slot_ptr(c, bound(static_cast<int>(c), total, ctas) >= u0 ? 0 : 1);
#pragma unroll
          for (int f = 0; f < 2 * kNT; ++f) q[k][f] = __ldcg(src + f);
        }
#pragma unroll
      for (int k = 0; k < kBatch; ++k)
        if (k0 + k < shares) {
#pragma unroll
          for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int n = 0; n < kNT; ++n) {
              const float4 w = q[k][i * kNT + n];
              v[i][n][0] += w.x; v[i][n][1] += w.y; v[i][n][2] += w.z; v[i][n][3] += w.w;
            }
        }
    }
    finish(tile, v);
  };
  // At the end of the share: when every other part of `tile` is already
  // counted, this CTA is the last without counting itself; it adds the parts
  // in CTA order with its own from registers (the sum the counting path
  // forms) and finishes the tile.  Otherwise it returns false.
  auto finish_if_complete = [&](int tile, const float (&own)[2][kNT][4]) -> bool {
    const int shares = shares_of(tile);
    uint32_t seen = 0;
    if (lane == 0) seen = ld_acquire_u32(a.cnt + static_cast<int64_t>(tile) * kConsumerWarps + warp);
    seen = __shfl_sync(0xFFFFFFFFu, seen, 0);
    if (static_cast<int>(seen) + 1 != shares) return false;
    __syncwarp();      // lane 0's acquire is ordered before every lane's slot reads
    float v[2][kNT][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int n = 0; n < kNT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) v[i][n][e] = 0.0f;
    const int64_t u0 = static_cast<int64_t>(tile) * steps;
    const int64_t c0 = owner_of(u0, total, ctas);
    for (int k = 0; k < shares; ++k) {
      const int64_t c = c0 + k;
      float4 q[2 * kNT];
      if (c == blockIdx.x) {
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int n = 0; n < kNT; ++n) q[i * kNT + n] = make_float4(own[i][n][0], own[i][n][1], own[i][n][2], own[i][n][3]);
      } else {
        const float4* src = slot_ptr(c, bound(static_cast<int>(c), total, ctas) >= u0 ? 0 : 1);
#pragma unroll
        for (int f = 0; f < 2 * kNT; ++f) q[f] = __ldcg(src + f);
      }
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int n = 0; n < kNT; ++n) {
          const float4 w = q[i * kNT + n];
          v[i][n][0] += w.x; v[i][n][1] += w.y; v[i][n][2] += w.z; v[i][n][3] += w.w;
        }
    }
    finish(tile, v);
    return true;
  };
  // LoRA B rows of a tile into L2 ahead of its finish (lane (g, t) takes row
  // group t of its rows, one 128-byte line per 64 rank columns)
  auto prefetch_b = [&](int tile) {
    // every lane walks the adapters (their list is shuffled across the warp);
    // only lanes with a row in the weight prefetch
    const int64_t row = static_cast<int64_t>(tile) * kRows + warp * 32 + 8 * t + pg;
    const bool in_w = row < a.nw;
    auto rows_of = [&](const uint16_t* lb) {
      if (!in_w) return;
      for (int grp = 0; grp < a.lora_steps; ++grp)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(lb + row * a.r + grp * 64));
    };
    if (a.adapter_idx == nullptr) rows_of(a.lora_b);
    else for_each_adapter([&](int ad) { rows_of(a.lora_b + static_cast<int64_t>(ad) * a.b_stride); });
  };

  float y[2][kNT][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int n = 0; n < kNT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) y[i][n][e] = 0.0f;
  // A first tile that ends within kDeferSteps steps of the start goes to slot 0
  // at once and is counted at the next tile end (or the end of the share),
  // when the previous kernel (X A^T slices, zeroed counters) has surely
  // finished, so the wait for it does not stall the stream.  A later first
  // tile end waits for that kernel (long done by then) and counts at once, so
  // that the share's end finds it counted.
  int pending = -1;
  bool dep_done = false;

  prefetch_b(first.tile);
  Pos pos = first;
  uint32_t s = 0, ph = 0;
  bool alive = true;
  for (int64_t it = 0; it < n_mine; ++it) {
    // the stage of this step: test first (cheap when the data is already there)
    if (!mbar_test_wait(&full[s], ph) && !mbar_wait(&full[s], ph, a.err)) { alive = false; break; }
    // this step's constants c[q][b] for the lane's rows warp*32 + 8q + pg
    float c[4][4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = lds128f(hole(32u * s + 4u * warp + q, static_cast<uint32_t>(pg) * 16u));
      c[q][0] = v.x; c[q][1] = v.y; c[q][2] = v.z; c[q][3] = v.w;
    }
    const uint32_t cs = code_stage(s) + crow;
    const uint32_t xs = xs0 + s * kXTile;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const uint32_t coff = ((((2u * b) + (t >> 1)) ^ pg) << 4) | ((t & 1u) << 3);
      uint2 cw[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) cw[q] = lds64(cs + q * 1024u + coff);
      uint4 xv[kNT][2];
#pragma unroll
      for (int n = 0; n < kNT; ++n)
#pragma unroll
        for (int jp = 0; jp < 2; ++jp) xv[n][jp] = lds128_if(xon[n], xs + b * kXBox + xoff[n][jp]);
      if (b == 3) {
        __syncwarp();
        mbar_arrive_if(lane == 0, &empty[s]);                 // stage fully read
      }
      float p[2][kNT][4];                                     // [m tile][n tile][element]
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t sel0 = 0x7604u | ((2u * (j & 1)) << 4);   // byte 2(j&1) of the word
        const uint32_t sel1 = sel0 + 0x10u;                      // byte 2(j&1) + 1
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const uint32_t w0 = (j < 2) ? cw[2 * i].x : cw[2 * i].y;
          const uint32_t w1 = (j < 2) ? cw[2 * i + 1].x : cw[2 * i + 1].y;
          const uint32_t a0 = lds_table(__byte_perm(w0, tbase, sel0));
          const uint32_t a1 = lds_table(__byte_perm(w1, tbase, sel0));
          const uint32_t a2 = lds_table(__byte_perm(w0, tbase, sel1));
          const uint32_t a3 = lds_table(__byte_perm(w1, tbase, sel1));
#pragma unroll
          for (int n = 0; n < kNT; ++n) {
            const uint32_t b0 = (j & 1) ? xv[n][j >> 1].z : xv[n][j >> 1].x;
            const uint32_t b1 = (j & 1) ? xv[n][j >> 1].w : xv[n][j >> 1].y;
            if (j == 0) mma_bf16_16816_z(p[i][n], a0, a1, a2, a3, b0, b1);
            else mma_bf16_16816(p[i][n], a0, a1, a2, a3, b0, b1);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int n = 0; n < kNT; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) y[i][n][e] = __fmaf_rn(c[2 * i + (e >> 1)][b], p[i][n][e], y[i][n][e]);
    }

    if (pos.step == steps - 1 || it == n_mine - 1) {
      // end of this CTA's part of the tile
      const bool last = it == n_mine - 1;
      const int shares = shares_of(pos.tile);
      if (!last) prefetch_b(pos.tile + 1);
      if (!dep_done && pending < 0 && !last && shares > 1 && it < kDeferSteps) {
        // so early that the previous kernel (X A^T slices, zeroed counters) may
        // still run: the partial waits in slot 0 and is counted later
        put_slot(0, y);
        pending = pos.tile;
      } else {
        if (!dep_done) {
          grid_dependency_wait();
          dep_done = true;
          stage_sxa();
          __syncwarp();
          if (lane == 0) mbar_arrive(xa_bar);
          if (!mbar_test_wait(xa_bar, 0) && !mbar_wait(xa_bar, 0, a.err)) { alive = false; break; }
        }
        if (pending >= 0) {
          float v[2][kNT][4];
          arrive(pending, v);
          pending = -1;
        }
        if (shares == 1) {
          finish(pos.tile, y);                                // no other CTA holds a part of it
        } else if (!(last && finish_if_complete(pos.tile, y))) {
          // slot 0 for the share's first tile, else 1 (a tile inside the share
          // is finished at once, so slot 1 is free again for the next one)
          put_slot(pos.tile == first.tile ? 0 : 1, y);
          arrive(pos.tile, y);
        }
      }
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int n = 0; n < kNT; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) y[i][n][e] = 0.0f;
    }
    pos = advance(pos);
    if (++s == kStages) { s = 0; ph ^= 1u; }
  }
  (void)alive;
}

// Partial X A^T and the zeroed tile counters of k_gemv.  CTA (c, sp) computes
// LoRA columns 4c .. 4c + 3 for every token over the sp-th of nsplit slices of
// K and writes them to part[sp] (no atomics, so nothing needs zeroing); k_gemv
// sums the slices when it first finishes a tile.  The CTA has a thread per
// 8-column chunk of its slice (a grid-stride loop covers longer slices), so
// the whole grid waits for about one load latency; warps reduce with shuffles
// and the warps' sums are added in warp order through shared memory, so the
// result does not depend on timing.  k_gemv, launched as the programmatic
// dependent of this grid, waits for it only before it first counts a tile.
// The four A rows' 8 columns of chunk ch, unpacked.
__device__ __forceinline__ void load_a_rows(const uint16_t* __restrict__ A, int j0, int r, int64_t kw,
                                            int64_t ch, float (&af)[4][8]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 v = (j0 + c < r) ? __ldg(reinterpret_cast<const uint4*>(A + (j0 + c) * kw) + ch)
                                 : make_uint4(0u, 0u, 0u, 0u);
    af[c][0] = bf16_lo(v.x); af[c][1] = bf16_hi(v.x); af[c][2] = bf16_lo(v.y); af[c][3] = bf16_hi(v.y);
    af[c][4] = bf16_lo(v.z); af[c][5] = bf16_hi(v.z); af[c][6] = bf16_lo(v.w); af[c][7] = bf16_hi(v.w);
  }
}

constexpr int kXaMaxThreads = 256;

// kMulti: every token has its own adapter (A + idx[i] * a_stride); its A rows
// are loaded per token.  Tokens without a valid adapter accumulate nothing.
template <int kMaxM, bool kMulti>
__global__ void __launch_bounds__(kXaMaxThreads)
k_xa_zero(const uint16_t* __restrict__ X, const uint16_t* __restrict__ A, int64_t m, int64_t kw, int r,
          float* __restrict__ part, int64_t ld, float4* __restrict__ zero4, int64_t n4,
          const int32_t* __restrict__ idx, int n_adapters, int64_t a_stride, uint32_t* err) {
  launch_dependents();
  __shared__ float s_red[kXaMaxThreads / 32][4 * kMaxM];
  const int mi = static_cast<int>(m);
  const int j0 = blockIdx.x * 4;
  const int64_t nch = kw / 8;
  const int64_t c_beg = (nch * blockIdx.y) / gridDim.y, c_end = (nch * (blockIdx.y + 1)) / gridDim.y;
  float acc[4][kMaxM];
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int i = 0; i < kMaxM; ++i) acc[c][i] = 0.0f;
  int ad[kMaxM];                           // kMulti: token i's adapter, -1 for none
  if constexpr (kMulti) {
    bool bad = false;
#pragma unroll
    for (int i = 0; i < kMaxM; ++i) {
      ad[i] = i < mi ? __ldg(idx + i) : -1;
      if (ad[i] >= n_adapters) { bad = true; ad[i] = -1; }
    }
    if (bad && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) atomicOr(err, kErrBadAdapter);
  }
  for (int64_t ch = c_beg + threadIdx.x; ch < c_end; ch += blockDim.x) {
    float af[4][8];
    if constexpr (!kMulti) {
      uint4 xv[kMaxM];                       // every load of the chunk issued before any use
#pragma unroll
      for (int i = 0; i < kMaxM; ++i)
        xv[i] = i < mi ? __ldg(reinterpret_cast<const uint4*>(X + i * kw) + ch) : make_uint4(0u, 0u, 0u, 0u);
      load_a_rows(A, j0, r, kw, ch, af);     // shared by every token
#pragma unroll
      for (int i = 0; i < kMaxM; ++i) {
        const float xf[8] = {bf16_lo(xv[i].x), bf16_hi(xv[i].x), bf16_lo(xv[i].y), bf16_hi(xv[i].y),
                             bf16_lo(xv[i].z), bf16_hi(xv[i].z), bf16_lo(xv[i].w), bf16_hi(xv[i].w)};
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[c][i] = __fmaf_rn(af[c][e], xf[e], acc[c][i]);
      }
    } else {
      // one token at a time: its own adapter's A rows and its X chunk
#pragma unroll
      for (int i = 0; i < kMaxM; ++i) {
        if (ad[i] < 0) continue;
        load_a_rows(A + static_cast<int64_t>(ad[i]) * a_stride, j0, r, kw, ch, af);
        const uint4 xv = __ldg(reinterpret_cast<const uint4*>(X + i * kw) + ch);
        const float xf[8] = {bf16_lo(xv.x), bf16_hi(xv.x), bf16_lo(xv.y), bf16_hi(xv.y),
                             bf16_lo(xv.z), bf16_hi(xv.z), bf16_lo(xv.w), bf16_hi(xv.w)};
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[c][i] = __fmaf_rn(af[c][e], xf[e], acc[c][i]);
      }
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = static_cast<int>(blockDim.x >> 5);
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int i = 0; i < kMaxM; ++i) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[c][i] += __shfl_xor_sync(0xFFFFFFFFu, acc[c][i], o);
    }
  if (lane == 0) {
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int i = 0; i < kMaxM; ++i) s_red[warp][c * kMaxM + i] = acc[c][i];
  }
  __syncthreads();
  // thread e < 4 kMaxM adds output e over the warps in order
  const int e = static_cast<int>(threadIdx.x);
  if (e < 4 * kMaxM) {
    const int c = e / kMaxM, i = e - (e / kMaxM) * kMaxM;
    float v = 0.0f;
    for (int w = 0; w < nwarps; ++w) v += s_red[w][e];
    if (i < mi && j0 + c < r) part[(static_cast<int64_t>(blockIdx.y) * 16 + i) * ld + j0 + c] = v;
  }
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * gridDim.y * blockDim.x;
  const int64_t gtid = (static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x) * blockDim.x + threadIdx.x;
  const float4 z = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  for (int64_t q = gtid; q < n4; q += nthreads) zero4[q] = z;
}

cudaError_t launch_pdl(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, void** args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelExC(&cfg, fn, args);
  if (e != cudaSuccess) (void)cudaGetLastError();   // leave no stale error for the next launch check
  return e;
}

template <int kNT, bool kQuad>
cudaError_t launch_gemv_t(const GemvArgs& args, const CUtensorMap& cm, const CUtensorMap& xm, int num_sms,
                          cudaStream_t stream) {
  static std::atomic<uint64_t> attr_done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_done.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(k_gemv<kNT, kQuad>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(GemvStages<kNT>::kSmemTop));
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(bit, std::memory_order_acq_rel);
  }
  // no more CTAs than steps, so that every CTA's share is non-empty
  const int64_t total = static_cast<int64_t>(args.m_tiles) * args.steps;
  int64_t grid64 = total < num_sms ? total : num_sms;
  if (grid64 > kMaxGemvCtas) grid64 = kMaxGemvCtas;
  const unsigned grid = static_cast<unsigned>(grid64);
  GemvArgs a = args;
  CUtensorMap c = cm, x = xm;
  void* kargs[3] = {&a, &c, &x};
  // dynamic shared memory up to the map's top covers any start address of the window
  return launch_pdl(reinterpret_cast<const void*>(k_gemv<kNT, kQuad>), dim3(grid), dim3(kGemvThreads),
                    GemvStages<kNT>::kSmemTop, stream, kargs);
}

}  // namespace

int gemv_tile_rows() { return kRows; }

int64_t gemv_slot_floats(int64_t m_tiles, int64_t steps) {
  int64_t ctas = m_tiles * steps;
  if (ctas > kMaxGemvCtas) ctas = kMaxGemvCtas;
  return ctas * 2 * kConsumerWarps * 32 * 16;
}

template <bool kMulti>
void launch_xa_zero_t(dim3 grid, unsigned threads, const uint16_t* X, const uint16_t* A, int64_t m, int64_t kw,
                      int r, float* part, int64_t ld, float4* z4, int64_t n4, const int32_t* idx, int n_ad,
                      int64_t a_stride, uint32_t* err, cudaStream_t stream) {
  if (m <= 1)
    k_xa_zero<1, kMulti><<<grid, threads, 0, stream>>>(X, A, m, kw, r, part, ld, z4, n4, idx, n_ad, a_stride, err);
  else if (m <= 4)
    k_xa_zero<4, kMulti><<<grid, threads, 0, stream>>>(X, A, m, kw, r, part, ld, z4, n4, idx, n_ad, a_stride, err);
  else if (m <= 8)
    k_xa_zero<8, kMulti><<<grid, threads, 0, stream>>>(X, A, m, kw, r, part, ld, z4, n4, idx, n_ad, a_stride, err);
  else
    k_xa_zero<16, kMulti><<<grid, threads, 0, stream>>>(X, A, m, kw, r, part, ld, z4, n4, idx, n_ad, a_stride, err);
}

cudaError_t launch_xa_zero(const uint16_t* X, const uint16_t* A, int64_t m, int64_t kw, int r, float* part,
                           int64_t ld, int splits, float* zero, int64_t n_zero, const int32_t* adapter_idx,
                           int n_adapters, int64_t a_stride, uint32_t* err, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>((r + 3) / 4), static_cast<unsigned>(splits));
  // a thread per chunk of the longest slice, in whole warps (at most
  // kXaMaxThreads): a thread that loads two chunks at once is slower
  const int64_t per_split = (kw / 8 + splits - 1) / splits;
  int64_t threads = (per_split + 31) / 32 * 32;
  if (threads > kXaMaxThreads) threads = kXaMaxThreads;
  if (threads < 64) threads = 64;
  float4* z4 = reinterpret_cast<float4*>(zero);
  const int64_t n4 = n_zero / 4;
  if (adapter_idx)
    launch_xa_zero_t<true>(grid, static_cast<unsigned>(threads), X, A, m, kw, r, part, ld, z4, n4, adapter_idx,
                           n_adapters, a_stride, err, stream);
  else
    launch_xa_zero_t<false>(grid, static_cast<unsigned>(threads), X, A, m, kw, r, part, ld, z4, n4, nullptr, 1,
                            0, err, stream);
  return cudaGetLastError();
}

int xa_splits_for(int r, int64_t kw) {
  // about 128 CTAs with a thread per 8-column chunk; more slices (up to the
  // most k_gemv sums) and threads when K is longer
  const int groups = (r + 3) / 4;
  const int64_t want = (kw / 8 + 127) / 128;  // slices of 128 chunks
  int64_t s = 128 / groups;
  if (s < want) s = want;
  if (s > kMaxXaSplits) s = kMaxXaSplits;
  if (s > (kw / 8) / 32) s = (kw / 8) / 32;   // at least a warp of chunks per slice
  return s < 1 ? 1 : static_cast<int>(s);
}

cudaError_t launch_gemv(const GemvArgs& args, const CUtensorMap& codes_map, const CUtensorMap& x_map,
                        int num_sms, cudaStream_t stream) {
  const bool quad = (args.kw / 64) % 4 == 0;
  if (args.m <= 8)
    return quad ? launch_gemv_t<1, true>(args, codes_map, x_map, num_sms, stream)
                : launch_gemv_t<1, false>(args, codes_map, x_map, num_sms, stream);
  return quad ? launch_gemv_t<2, true>(args, codes_map, x_map, num_sms, stream)
              : launch_gemv_t<2, false>(args, codes_map, x_map, num_sms, stream);
}

}  // namespace qlora
