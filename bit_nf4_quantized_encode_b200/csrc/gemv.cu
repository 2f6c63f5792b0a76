// gemv.cu -- decode-shaped forward of the NF4 LoRA linear layer (M <= 16 tokens).
//
// Y = X deq(W)^T + s (X A^T) B^T with few token rows is a stream over the packed
// weight (automatone "QLoRA paper explained", section "How it works": the 4-bit
// weight is dequantized on the fly for the matmul), bound by HBM.  Three
// kernels, each launched as the programmatic dependent of the one before it:
//
// k_xa_zero: partial X A^T over slices of K in fp32 (CUDA cores, CTAs that fit
//   beside k_gemv's) and the zeroed fp32 split buffer of k_gemv.
//
// k_gemv: the weight stream.  Each CTA takes an equal, contiguous share of all
//   (256-row tile, 256-column step) pairs, so the work is balanced whatever the
//   shape; a CTA adds its fp32 partial of each tile it touched to the split
//   buffer with atomics, and at its end sums its share of the X A^T slices.
//   * Thread 0 streams the [256 rows x 128 bytes] code tile (128B-swizzled) and
//     the four [m x 64] activation boxes of each step into a 3-deep ring (TMA).
//   * 16 / kMT warps own 16 kMT weight rows each.  For every 64-column block
//     they read their rows' code bytes, turn each byte into the two bf16 levels
//     it encodes with one shared-memory load from a 256-entry pair table (one
//     copy per lane: conflict-free), and feed them straight from registers to
//     warp MMAs (m16n8k16, bf16 in, fp32 out): a code byte is exactly one
//     A-fragment register.  The block's product is scaled by its constant
//     c1' = fma(e4m3(q), c2/448, mu) and added to fp32 registers.
//   * The tensor core here only replaces FMAs: per weight it does 2 M FLOP.
//     Warp MMAs are used because a skinny-N product issued as tcgen05.mma
//     from one thread costs about 80 cycles per 128x16x16 instruction, which
//     caps a 16-token stream near 25 weights per cycle per SM, while HBM
//     delivers about 46.
//
// k_finish: Y = bf16(split + s (X A^T) B^T), one thread per weight row.
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
__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
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

// Block-constant inputs of one step for one weight row, loaded ahead: the E4M3
// bytes of the step's four blocks (byte b = block b) and c2 of the first
// block's group (and, when K is not a multiple of 256 columns, of the last
// block's group too).
struct RowConsts {
  uint32_t q;
  float c2a, c2b;
};

// kMT m16 tiles (16 kMT weight rows) per warp, 16 / kMT warps per CTA.
template <int kMT>
struct GemvShape {
  static constexpr int kWarps = 16 / kMT;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kRowsPerWarp = 16 * kMT;
  static constexpr int kMaxRegs = kMT == 1 ? 112 : 224;
};

template <int kNT, bool kQuad, int kMT>   // kNT: n8 token tiles (1: M <= 8, 2: M <= 16); kQuad: K % 256 == 0
__global__ void __maxnreg__(GemvShape<kMT>::kMaxRegs)
k_gemv(const GemvArgs a, const __grid_constant__ CUtensorMap cmap,
       const __grid_constant__ CUtensorMap xmap) {
  using S = GemvShape<kMT>;
  constexpr int kWarps = S::kWarps;
  constexpr int kThreads = S::kThreads;
  constexpr int kRW = S::kRowsPerWarp;
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
  uint64_t* full = bars;                  // codes + X landed (TMA)
  uint64_t* empty = bars + kStages;       // one arrival per warp
  float* s_level = reinterpret_cast<float*>(gptr(misc + 64));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t steps = a.steps;
  const int64_t total = static_cast<int64_t>(a.m_tiles) * steps;
  const int64_t x_beg = bound(blockIdx.x, total, gridDim.x);
  const int64_t x_end = bound(blockIdx.x + 1, total, gridDim.x);
  const int kblocks = static_cast<int>(a.kw / 64);
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

  // TMA issue (thread 0): iteration i goes to stage i % kStages once every warp
  // has released that stage's previous iteration.
  const uint32_t xbytes = 4u * static_cast<uint32_t>(m) * 128u;
  const bool producer = threadIdx.x == 0;
  Pos ppos = first;
  int64_t pit = 0;
  uint32_t ps = 0, pph = 0;
  // issue the next step if its stage is free; `block` waits (bounded) for it
  auto issue_next = [&](bool block) -> bool {
    if (pit >= n_mine) return true;
    if (!mbar_test_wait(&empty[ps], pph ^ 1u)) {
      if (!block) return true;
      if (!mbar_wait(&empty[ps], pph ^ 1u, a.err)) return false;
    }
    mbar_arrive_expect_tx(&full[ps], kCodeTile + xbytes);
    const int col0 = ppos.step * kStepCols;
    tma_load_2d(gptr(code_stage(ps)), &cmap, col0 / 2, ppos.tile * kRows, &full[ps]);
#pragma unroll
    for (int b = 0; b < 4; ++b)
      tma_load_2d(gptr(xs0 + ps * kXTile + b * kXBox), &xmap, col0 + b * 64, 0, &full[ps]);
    ppos = advance(ppos);
    ++pit;
    if (++ps == kStages) { ps = 0; pph ^= 1u; }
    return true;
  };
  if (producer) {
    tma_prefetch_desc(&cmap);
    tma_prefetch_desc(&xmap);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kWarps);
    }
    fence_barrier_init();
  }

  // ------------------------------------------------ compute
  // Lane (g, t) serves MMA rows g and g + 8 of the warp's kMT m16 tiles.  MMA
  // row g of an 8-row group is weight row 8u + pg with pg = 2(g mod 4) + g / 4,
  // so that the lanes of each half-warp read rows whose 128-byte swizzle
  // patterns differ in bits 1 and 2 (no bank conflicts).  The lane's rows are
  // warp*16kMT + 8q + pg (q < 2kMT; tile i uses q = 2i and 2i + 1).  In every
  // 64-column block the lane reads the code bytes [8t, 8t + 8) of those rows.
  // Columns enter the MMA in a permuted order (the same for X): slice j of a
  // block feeds columns 16t + 4j + {0, 1} as k = {2t, 2t+1} and 16t + 4j + {2, 3}
  // as k = {2t+8, 2t+9}, so every lane reads only its own bytes.
  //
  // Block constants: lane L computes the constants of weight row
  // warp*16kMT + (L mod 16kMT) (all four blocks when kMT = 2, blocks
  // 2(L / 16) and 2(L / 16) + 1 when kMT = 1) and stores them in a two-slot
  // table in the free halves of pair-table rows 0..63; the lanes that read them
  // belong to the same warp.
  const int g = lane >> 2, t = lane & 3;
  const int pg = ((g & 3) << 1) | (g >> 2);
  const uint32_t tbase = kTableAddr | (static_cast<uint32_t>(lane) << 2);
  const uint32_t crow = static_cast<uint32_t>(warp * kRW + pg) * 128u;
  const float mu = __ldg(a.mean);
  const uint32_t kbl = static_cast<uint32_t>(kblocks);

  const int crow_l = warp * kRW + (lane & (kRW - 1));          // this lane's constant row
  const int cb0 = kMT == 2 ? 0 : 2 * (lane >> 4);              // its first block
  auto cblk0 = [&](Pos p) -> uint32_t {                        // block indices < 2^32
    return static_cast<uint32_t>(p.tile * kRows + crow_l) * kbl + 4u * p.step;
  };
  auto load_raw = [&](Pos p, bool valid, RowConsts& k) {
    k.q = 0;
    k.c2a = 0.0f;
    k.c2b = 0.0f;
    if (valid && p.tile * kRows + crow_l < a.nw) {
      const uint32_t blk0 = cblk0(p);
      if (kQuad) {
        k.q = __ldg(reinterpret_cast<const uint32_t*>(a.qabs + blk0));
        k.c2a = __ldg(a.c2 + (blk0 >> 8));
      } else {
        const int nb = min(4, kblocks - 4 * p.step);
#pragma unroll
        for (int b = 0; b < 4; ++b)
          if (b < nb) k.q |= static_cast<uint32_t>(__ldg(a.qabs + blk0 + b)) << (8 * b);
        k.c2a = __ldg(a.c2 + (blk0 >> 8));
        k.c2b = __ldg(a.c2 + ((blk0 + nb - 1) >> 8));
      }
    }
  };
  uint32_t grp_cache = 0xFFFFFFFFu;
  float c2q_cache = 0.0f;
  // c[b] = fma(e4m3(q_b), c2 / 448, mu) for the lane's row and blocks, into slot `slot`
  auto write_consts = [&](Pos p, const RowConsts& k, uint32_t slot) {
    const uint32_t blk0 = cblk0(p);
    const uint32_t grp = blk0 >> 8;
    if (grp != grp_cache) {
      grp_cache = grp;
      c2q_cache = __fdiv_rn(k.c2a, 448.0f);
    }
    float f[4];
    e4m3x4_to_f32(k.q, f);
    float c[4];
    if (kQuad) {
#pragma unroll
      for (int b = 0; b < 4; ++b) c[b] = __fmaf_rn(f[b], c2q_cache, mu);
    } else {
      const float c2q_b = __fdiv_rn(k.c2b, 448.0f);
#pragma unroll
      for (int b = 0; b < 4; ++b) c[b] = __fmaf_rn(f[b], ((blk0 + b) >> 8) == grp ? c2q_cache : c2q_b, mu);
    }
    const uint32_t e = slot * 256u + static_cast<uint32_t>(crow_l);
    if (kMT == 2) {
      sts128(hole(e >> 3, (e & 7u) * 16u), c[0], c[1], c[2], c[3]);
    } else {
      const float c0 = cb0 == 0 ? c[0] : c[2], c1 = cb0 == 0 ? c[1] : c[3];
      asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(hole(e >> 3, (e & 7u) * 16u + cb0 * 4u)),
                   "f"(c0), "f"(c1) : "memory");
    }
  };

  Pos pos = first;
  Pos pos1 = advance(pos), pos2 = advance(pos1), pos3 = advance(pos2);
  RowConsts r0, ra, rb;                   // raw inputs of steps 0, it + 1 and it + 2
  load_raw(pos, n_mine > 0, r0);
  load_raw(pos1, n_mine > 1, ra);
  load_raw(pos2, n_mine > 2, rb);

  if (threadIdx.x < 16) s_level[threadIdx.x] = a.level[threadIdx.x];
  __syncthreads();                        // levels, barrier initialisation
  // the first loads are in flight while the pair table is built
  if (producer)
    for (int i = 0; i < kStages - 1; ++i) issue_next(true);
  // pair table: entry (byte v, lane l) = {bf16(L[v >> 4]), bf16(L[v & 15])}, element order;
  // thread v converts entry v once and writes its 32 copies
  for (int v = threadIdx.x; v < 256; v += kThreads) {
    const __nv_bfloat162 e = __floats2bfloat162_rn(s_level[v >> 4], s_level[v & 15]);
    const float ev = __uint_as_float(*reinterpret_cast<const uint32_t*>(&e));
#pragma unroll
    for (int l = 0; l < 32; l += 4) sts128(kTableAddr + v * 256 + l * 4, ev, ev, ev, ev);
  }
  write_consts(pos, r0, 0);
  __syncthreads();                        // pair table and step 0's constants in place
  launch_dependents();                    // k_finish may be scheduled; it waits for this grid

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

  float y[kMT][kNT][4];
#pragma unroll
  for (int i = 0; i < kMT; ++i)
#pragma unroll
    for (int n = 0; n < kNT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) y[i][n][e] = 0.0f;
  // The partial of the first tile this CTA touches is kept in registers until
  // the next tile boundary (or the end of the range): by then the previous
  // kernel (X A^T and the zeroed split buffer) has surely finished, so the wait
  // for it does not stall the stream.
  float ys[kMT][kNT][4];
  int ys_tile = -1;
  bool dep_done = false;
  // add a tile partial to the split buffer (fire-and-forget reductions)
  auto flush = [&](int tile, float (&v)[kMT][kNT][4]) {
#pragma unroll
    for (int i = 0; i < kMT; ++i)
#pragma unroll
      for (int n = 0; n < kNT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int64_t row = static_cast<int64_t>(tile) * kRows + warp * kRW + 8 * (2 * i + (e >> 1)) + pg;
          const int tok = 8 * n + 2 * t + (e & 1);
          if (row < a.nw && tok < m) atomicAdd(a.yacc + tok * a.nw + row, v[i][n][e]);
        }
  };

  uint32_t s = 0, ph = 0;
  bool alive = true;
  for (int64_t it = 0; it < n_mine && alive; ++it) {
    // this step's constants c[q][b] for the lane's rows warp*16kMT + 8q + pg
    float c[2 * kMT][4];
    const uint32_t cslot = static_cast<uint32_t>(it & 1) * 256u;
#pragma unroll
    for (int q = 0; q < 2 * kMT; ++q) {
      const uint32_t e = cslot + static_cast<uint32_t>(warp * kRW + 8 * q + pg);
      const float4 v = lds128f(hole(e >> 3, (e & 7u) * 16u));
      c[q][0] = v.x; c[q][1] = v.y; c[q][2] = v.z; c[q][3] = v.w;
    }
    // the stage of this step: test first (cheap when the data is already there)
    if (!mbar_test_wait(&full[s], ph) && !mbar_wait(&full[s], ph, a.err)) break;
    const uint32_t cs = code_stage(s) + crow;
    const uint32_t xs = xs0 + s * kXTile;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const uint32_t coff = ((((2u * b) + (t >> 1)) ^ pg) << 4) | ((t & 1u) << 3);
      uint2 cw[2 * kMT];
#pragma unroll
      for (int q = 0; q < 2 * kMT; ++q) cw[q] = lds64(cs + q * 1024u + coff);
      uint4 xv[kNT][2];
#pragma unroll
      for (int n = 0; n < kNT; ++n)
#pragma unroll
        for (int jp = 0; jp < 2; ++jp) xv[n][jp] = lds128_if(xon[n], xs + b * kXBox + xoff[n][jp]);
      if (b == 3) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);                // stage fully read
      }
      if (b == 1) {
        // next step's constants into the other slot (read two steps ago by
        // this warp; the syncwarp at b == 3 orders them before their readers)
        __syncwarp();
        if (it + 1 < n_mine) write_consts(pos1, ra, static_cast<uint32_t>((it + 1) & 1));
      }
      if (producer && !issue_next(b == 3)) { alive = false; break; }
      float p[kMT][kNT][4];                                   // [m tile][n tile][element]
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t sel0 = 0x7604u | ((2u * (j & 1)) << 4);   // byte 2(j&1) of the word
        const uint32_t sel1 = sel0 + 0x10u;                      // byte 2(j&1) + 1
#pragma unroll
        for (int i = 0; i < kMT; ++i) {
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
      for (int i = 0; i < kMT; ++i)
#pragma unroll
        for (int n = 0; n < kNT; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) y[i][n][e] = __fmaf_rn(c[2 * i + (e >> 1)][b], p[i][n][e], y[i][n][e]);
    }
    if (!alive) break;

    if (pos.step == steps - 1 || it == n_mine - 1) {
      // end of this CTA's share of the tile
      if (!dep_done && ys_tile < 0 && it != n_mine - 1) {
        ys_tile = pos.tile;                                   // keep it for later
#pragma unroll
        for (int i = 0; i < kMT; ++i)
#pragma unroll
          for (int n = 0; n < kNT; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) ys[i][n][e] = y[i][n][e];
      } else {
        if (!dep_done) {
          grid_dependency_wait();
          dep_done = true;
        }
        if (ys_tile >= 0) {
          flush(ys_tile, ys);
          ys_tile = -1;
        }
        flush(pos.tile, y);
      }
#pragma unroll
      for (int i = 0; i < kMT; ++i)
#pragma unroll
        for (int n = 0; n < kNT; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) y[i][n][e] = 0.0f;
    }
    ra = rb;                                   // loaded a full step ago
    load_raw(pos3, it + 3 < n_mine, rb);
    pos = pos1; pos1 = pos2; pos2 = pos3; pos3 = advance(pos3);
    if (++s == kStages) { s = 0; ph ^= 1u; }
  }
  if (!alive) return;
  // this CTA's share of X A^T: the sum of k_xa_zero's K slices (complete once
  // the wait above has returned; every CTA reached it at its last flush)
  {
    const int nxa = m * a.r;
    const int e_beg = static_cast<int>((static_cast<int64_t>(nxa) * blockIdx.x) / gridDim.x);
    const int e_end = static_cast<int>((static_cast<int64_t>(nxa) * (blockIdx.x + 1)) / gridDim.x);
    for (int e = e_beg + static_cast<int>(threadIdx.x); e < e_end; e += kThreads) {
      const int i = e / a.r, j = e - (e / a.r) * a.r;
      float v = 0.0f;
      for (int sp = 0; sp < a.xa_splits; ++sp) v += __ldcg(a.xa_part + (static_cast<int64_t>(sp) * 16 + i) * a.ld_xa + j);
      a.xa[i * a.ld_xa + j] = v;
    }
  }
}

// Partial X A^T and the zeroed split buffer of k_gemv.  CTA (c, sp) computes
// LoRA columns 4c .. 4c + 3 for every token over the sp-th of nsplit slices of
// K and writes them to part[sp] (no atomics, so nothing needs zeroing); k_gemv
// sums the slices at its end.  Each of the 64 threads takes 8-column chunks a
// block stride apart; the CTA reduces with warp shuffles and one exchange
// through shared memory.  64 threads of at most 128 registers, so that a CTA
// fits beside a k_gemv CTA on one SM: k_gemv, launched as the programmatic
// dependent of this grid, starts streaming at once and only waits for it
// before its first atomic.
template <int kMaxM>
__global__ void __launch_bounds__(64, 8)
k_xa_zero(const uint16_t* __restrict__ X, const uint16_t* __restrict__ A, int64_t m, int64_t kw, int r,
          float* __restrict__ part, int64_t ld, float4* __restrict__ zero4, int64_t n4) {
  launch_dependents();
  __shared__ float s_red[4 * kMaxM];
  const int mi = static_cast<int>(m);
  const int j0 = blockIdx.x * 4;
  const int64_t nch = kw / 8;
  const int64_t c_beg = (nch * blockIdx.y) / gridDim.y, c_end = (nch * (blockIdx.y + 1)) / gridDim.y;
  float acc[4][kMaxM];
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int i = 0; i < kMaxM; ++i) acc[c][i] = 0.0f;
  for (int64_t ch = c_beg + threadIdx.x; ch < c_end; ch += blockDim.x) {
    float af[4][8];                        // the four A rows' 8 columns, unpacked once
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = (j0 + c < r) ? __ldg(reinterpret_cast<const uint4*>(A + (j0 + c) * kw) + ch)
                                   : make_uint4(0u, 0u, 0u, 0u);
      af[c][0] = bf16_lo(v.x); af[c][1] = bf16_hi(v.x); af[c][2] = bf16_lo(v.y); af[c][3] = bf16_hi(v.y);
      af[c][4] = bf16_lo(v.z); af[c][5] = bf16_hi(v.z); af[c][6] = bf16_lo(v.w); af[c][7] = bf16_hi(v.w);
    }
    uint4 xv[kMaxM];
#pragma unroll
    for (int i = 0; i < kMaxM; ++i)
      xv[i] = i < mi ? __ldg(reinterpret_cast<const uint4*>(X + i * kw) + ch) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int i = 0; i < kMaxM; ++i) {
      const float xf[8] = {bf16_lo(xv[i].x), bf16_hi(xv[i].x), bf16_lo(xv[i].y), bf16_hi(xv[i].y),
                           bf16_lo(xv[i].z), bf16_hi(xv[i].z), bf16_lo(xv[i].w), bf16_hi(xv[i].w)};
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[c][i] = __fmaf_rn(af[c][e], xf[e], acc[c][i]);
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int i = 0; i < kMaxM; ++i) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[c][i] += __shfl_xor_sync(0xFFFFFFFFu, acc[c][i], o);
    }
  if (warp == 1 && lane == 0) {
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int i = 0; i < kMaxM; ++i) s_red[c * kMaxM + i] = acc[c][i];
  }
  __syncthreads();
  if (warp == 0 && lane == 0) {
    float* dst = part + static_cast<int64_t>(blockIdx.y) * 16 * ld;
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int i = 0; i < kMaxM; ++i)
        if (i < mi && j0 + c < r) dst[i * ld + j0 + c] = acc[c][i] + s_red[c * kMaxM + i];
  }
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * gridDim.y * blockDim.x;
  const int64_t gtid = (static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x) * blockDim.x + threadIdx.x;
  const float4 z = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  for (int64_t e = gtid; e < n4; e += nthreads) zero4[e] = z;
}

// Y[i, n] = bf16(split[i, n] + s * sum_c XA[i, c] B[n, c]).  Four lanes per
// row n: lane q of the four takes the 8-column chunks cc = q, q + 4, ... of the
// rank, the four partial sums are combined with two butterfly shuffles, and
// lane q stores the tokens i = q, q + 4, ...  kMaxM (1, 4, 8 or 16) bounds the
// token count at compile time.
template <int kMaxM>
__global__ void __launch_bounds__(128)
k_finish(const float* __restrict__ yacc, const float* __restrict__ xa, int64_t ld_xa,
         const uint16_t* __restrict__ lora_b, int r, float s, int64_t m, int64_t nw, uint16_t* __restrict__ y,
         float* __restrict__ xa_out) {
  __shared__ __align__(16) float s_xa[kMaxM * 256];
  grid_dependency_wait();                  // k_gemv complete (it waited for k_xa_zero)
  const int mi = static_cast<int>(m);
  // X A^T into shared memory (row i at i * r)
  for (int j = threadIdx.x; j < r; j += blockDim.x) {
    float v[kMaxM];
#pragma unroll
    for (int i = 0; i < kMaxM; ++i) v[i] = i < mi ? __ldcg(xa + i * ld_xa + j) : 0.0f;
#pragma unroll
    for (int i = 0; i < kMaxM; ++i)
      if (i < mi) {
        s_xa[i * r + j] = v[i];
        if (xa_out && blockIdx.x == 0) xa_out[i * r + j] = v[i];
      }
  }
  const int q = threadIdx.x & 3;
  const int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 4) + (threadIdx.x >> 2);
  const bool live = n < nw;                // all lanes stay for the shuffles
  // split-buffer values of this lane's tokens and its first B chunks are issued
  // before the barrier, with the staging loads: one memory round trip per row
  constexpr int kMine = (kMaxM + 3) / 4;   // tokens stored by this lane
  float acc[kMine];
#pragma unroll
  for (int u = 0; u < kMine; ++u) {
    const int i = q + 4 * u;
    acc[u] = (live && i < mi) ? __ldcg(yacc + i * nw + n) : 0.0f;
  }
  const uint4* brow = reinterpret_cast<const uint4*>(lora_b + (live ? n : 0) * r);
  const int nch = r / 8;
  uint4 bv[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) bv[u] = (live && q + 4 * u < nch) ? __ldg(brow + q + 4 * u) : make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();                         // X A^T staged
  float lo[kMaxM];
#pragma unroll
  for (int i = 0; i < kMaxM; ++i) lo[i] = 0.0f;
  for (int c0 = q; c0 < nch; c0 += 16) {   // four chunks of eight rank columns per round
    if (c0 != q) {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        bv[u] = (live && c0 + 4 * u < nch) ? __ldg(brow + c0 + 4 * u) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int cc = c0 + 4 * u;
      if (cc >= nch) break;
      const float b8[8] = {bf16_lo(bv[u].x), bf16_hi(bv[u].x), bf16_lo(bv[u].y), bf16_hi(bv[u].y),
                           bf16_lo(bv[u].z), bf16_hi(bv[u].z), bf16_lo(bv[u].w), bf16_hi(bv[u].w)};
#pragma unroll
      for (int i = 0; i < kMaxM; ++i)
        if (i < mi) {
          const float4 x0 = *reinterpret_cast<const float4*>(&s_xa[i * r + cc * 8]);
          const float4 x1 = *reinterpret_cast<const float4*>(&s_xa[i * r + cc * 8 + 4]);
          float v = lo[i];
          v = __fmaf_rn(x0.x, b8[0], v); v = __fmaf_rn(x0.y, b8[1], v);
          v = __fmaf_rn(x0.z, b8[2], v); v = __fmaf_rn(x0.w, b8[3], v);
          v = __fmaf_rn(x1.x, b8[4], v); v = __fmaf_rn(x1.y, b8[5], v);
          v = __fmaf_rn(x1.z, b8[6], v); v = __fmaf_rn(x1.w, b8[7], v);
          lo[i] = v;
        }
    }
  }
#pragma unroll
  for (int i = 0; i < kMaxM; ++i) {
    lo[i] += __shfl_xor_sync(0xFFFFFFFFu, lo[i], 1);
    lo[i] += __shfl_xor_sync(0xFFFFFFFFu, lo[i], 2);
  }
  if (!live) return;
#pragma unroll
  for (int u = 0; u < kMine; ++u) {
    const int i = q + 4 * u;
    float v = lo[0];                         // lo[i] with compile-time indices
#pragma unroll
    for (int k = 1; k < kMaxM; ++k)
      if (k == i) v = lo[k];
    if (i < mi) {
      const __nv_bfloat16 h = __float2bfloat16_rn(__fmaf_rn(s, v, acc[u]));
      y[i * nw + n] = *reinterpret_cast<const uint16_t*>(&h);
    }
  }
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
  return cudaLaunchKernelExC(&cfg, fn, args);
}

template <int kNT, bool kQuad, int kMT>
cudaError_t launch_gemv_t(const GemvArgs& args, const CUtensorMap& cm, const CUtensorMap& xm, int num_sms,
                          cudaStream_t stream) {
  static std::atomic<uint64_t> attr_done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_done.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(k_gemv<kNT, kQuad, kMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(GemvStages<kNT>::kSmemTop));
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(bit, std::memory_order_acq_rel);
  }
  const int64_t total = static_cast<int64_t>(args.m_tiles) * args.steps;
  const unsigned grid = static_cast<unsigned>(total < num_sms ? total : num_sms);
  GemvArgs a = args;
  CUtensorMap c = cm, x = xm;
  void* kargs[3] = {&a, &c, &x};
  // dynamic shared memory up to the map's top covers any start address of the window
  return launch_pdl(reinterpret_cast<const void*>(k_gemv<kNT, kQuad, kMT>), dim3(grid),
                    dim3(GemvShape<kMT>::kThreads), GemvStages<kNT>::kSmemTop, stream, kargs);
}

template <int kMT>
cudaError_t launch_gemv_mt(const GemvArgs& args, const CUtensorMap& cm, const CUtensorMap& xm, int num_sms,
                           cudaStream_t stream) {
  const bool quad = (args.kw / 64) % 4 == 0;
  if (args.m <= 8)
    return quad ? launch_gemv_t<1, true, kMT>(args, cm, xm, num_sms, stream)
                : launch_gemv_t<1, false, kMT>(args, cm, xm, num_sms, stream);
  return quad ? launch_gemv_t<2, true, kMT>(args, cm, xm, num_sms, stream)
              : launch_gemv_t<2, false, kMT>(args, cm, xm, num_sms, stream);
}

}  // namespace

int gemv_tile_rows() { return kRows; }

cudaError_t launch_xa_zero(const uint16_t* X, const uint16_t* A, int64_t m, int64_t kw, int r, float* part,
                           int64_t ld, int splits, float* zero, int64_t n_zero, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>((r + 3) / 4), static_cast<unsigned>(splits));
  float4* z4 = reinterpret_cast<float4*>(zero);
  const int64_t n4 = n_zero / 4;
  if (m <= 1) k_xa_zero<1><<<grid, 64, 0, stream>>>(X, A, m, kw, r, part, ld, z4, n4);
  else if (m <= 4) k_xa_zero<4><<<grid, 64, 0, stream>>>(X, A, m, kw, r, part, ld, z4, n4);
  else if (m <= 8) k_xa_zero<8><<<grid, 64, 0, stream>>>(X, A, m, kw, r, part, ld, z4, n4);
  else k_xa_zero<16><<<grid, 64, 0, stream>>>(X, A, m, kw, r, part, ld, z4, n4);
  return cudaGetLastError();
}

int xa_splits_for(int r, int64_t kw) {
  const int groups = (r + 3) / 4;
  int s = 128 / groups;                       // about 128 CTAs in all
  const int64_t max_by_k = (kw / 8) / 64;     // at least one chunk per thread
  if (s > max_by_k) s = static_cast<int>(max_by_k);
  if (s > kMaxXaSplits) s = kMaxXaSplits;
  return s < 1 ? 1 : s;
}

cudaError_t launch_gemv(const GemvArgs& args, const CUtensorMap& codes_map, const CUtensorMap& x_map,
                        int num_sms, cudaStream_t stream) {
#ifdef GEMV_FORCE_MT
  return launch_gemv_mt<GEMV_FORCE_MT>(args, codes_map, x_map, num_sms, stream);
#else
  return launch_gemv_mt<2>(args, codes_map, x_map, num_sms, stream);
#endif
}

cudaError_t launch_gemv_finish(const float* yacc, const float* xa, int64_t ld_xa, const uint16_t* lora_b, int r,
                               float s, int64_t m, int64_t nw, uint16_t* y, float* xa_out, cudaStream_t stream) {
  void* kargs[10] = {&yacc, &xa, &ld_xa, &lora_b, &r, &s, &m, &nw, &y, &xa_out};
  const unsigned grid = static_cast<unsigned>((nw + 31) / 32);      // 32 rows per 128-thread CTA
  const void* fn = m <= 1 ? reinterpret_cast<const void*>(k_finish<1>)
                 : m <= 4 ? reinterpret_cast<const void*>(k_finish<4>)
                 : m <= 8 ? reinterpret_cast<const void*>(k_finish<8>)
                          : reinterpret_cast<const void*>(k_finish<16>);
  return launch_pdl(fn, dim3(grid), dim3(128), 0, stream, kargs);
}

}  // namespace qlora
