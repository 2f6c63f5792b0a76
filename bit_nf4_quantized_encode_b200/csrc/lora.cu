// lora.cu -- the rank-r contractions of the LoRA branch on tcgen05 / TMEM / TMA.
//
// What is computed (QLoRA, arXiv:2305.14314; automatone "QLoRA paper
// explained", section "How it works": the 16-bit LoRA adapters sit beside the
// frozen 4-bit weight, and the gradients land only on them):
//   forward   XA = X A^T                          [M, r]  (contraction over K)
//   backward  G  = dY B                           [M, r]  (contraction over N)
//             dB = dY^T (s XA)                    [N, r]  (contraction over the tokens)
//             dA = ((s G)^T X) = (X^T (s G))^T    [r, K]  (contraction over the tokens)
// Each is D[mdim, ndim] = P Q^T with the long operand P streamed once by TMA
// and the rank-r operand Q (small, L2-resident) beside it; ndim = r <= 256.
//
// One launch runs up to two such problems (XA with G; dB with dA), each cut
// into (128-row tile, 64-column tile, K split) units spread over a persistent
// grid.  A problem whose tiles alone would not fill the GPU splits its
// contraction; the partial tiles then go to slots in global memory and the
// unit that completes a tile's count (an atomic counter) sums the slots in
// split order, so every result is bit-reproducible from run to run -- no fp32
// atomics anywhere.  The epilogue writes any of: the fp32 result (optionally
// transposed, for dA), and bf16(scale * result) zero-padded to a multiple of
// 64 columns (the rank-r operand of the fused dequant-GEMM and of the next
// contraction), so no separate convert kernel runs.  A side job converts a
// caller-supplied fp32 X A^T to bf16(s X A^T) the same way.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "lora.h"
#include "sm100_ptx.cuh"

namespace qlora {
namespace {

constexpr int kStages = 6;
constexpr int kABytes = 128 * 128;     // 128 x 64 bf16
constexpr int kBBytes = 64 * 128;      // 64 x 64 bf16
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 6 * 32;       // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr uint32_t kTmemCols = 128;    // two 64-column accumulators
constexpr size_t kSmem = 1024 + kStages * kStageBytes + 256;

struct UnitPos {
  int prob, mt, nt, sp, kbeg, nk;
};

__device__ __forceinline__ UnitPos unit_pos(const RankArgs& a, int u) {
  UnitPos w;
  w.prob = (a.nprob > 1 && u >= a.p[1].unit_begin) ? 1 : 0;
  const RankProblem& p = a.p[w.prob];
  const int local = u - p.unit_begin;
  w.sp = local % p.splits;
  const int rest = local / p.splits;
  w.nt = rest % p.n_tiles;
  w.mt = rest / p.n_tiles;
  w.kbeg = static_cast<int>((static_cast<int64_t>(p.ksteps) * w.sp) / p.splits);
  w.nk = static_cast<int>((static_cast<int64_t>(p.ksteps) * (w.sp + 1)) / p.splits) - w.kbeg;
  return w;
}


__device__ __forceinline__ float4 ld_cg4(const float* p) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// The final values of row `row`, columns c0 .. c0 + 63 of problem p's D.
__device__ __forceinline__ void store_final(const RankProblem& p, int64_t row, int64_t c0, const float (&v)[64]) {
  if (row >= p.mdim) return;
  if (p.out_f32) {
    if (p.transpose) {                      // out[j * ld + row]: lanes walk rows, coalesced per column
#pragma unroll
      for (int c = 0; c < 64; ++c)
        if (c0 + c < p.ndim) p.out_f32[(c0 + c) * p.ld_f32 + row] = v[c];
    } else {
      float* dst = p.out_f32 + row * p.ld_f32 + c0;
#pragma unroll
      for (int c = 0; c < 64; c += 4)       // ndim and ld are multiples of 8: whole 16-byte pieces
        if (c0 + c < p.ndim) *reinterpret_cast<float4*>(dst + c) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
    }
  }
  if (p.out_bf16) {
    uint16_t* dst = p.out_bf16 + row * p.ld_bf16 + c0;
#pragma unroll
    for (int c = 0; c < 64; c += 8)
      if (c0 + c < p.bf16_cols) {           // columns past ndim hold zeros (zero-filled operand)
        const float s = p.bf16_scale;
        uint4 q;
        q.x = pack_bf16x2(__fmul_rn(s, v[c]), __fmul_rn(s, v[c + 1]));
        q.y = pack_bf16x2(__fmul_rn(s, v[c + 2]), __fmul_rn(s, v[c + 3]));
        q.z = pack_bf16x2(__fmul_rn(s, v[c + 4]), __fmul_rn(s, v[c + 5]));
        q.w = pack_bf16x2(__fmul_rn(s, v[c + 6]), __fmul_rn(s, v[c + 7]));
        *reinterpret_cast<uint4*>(dst + c) = q;
      }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
k_rank(const RankArgs a, const __grid_constant__ CUtensorMap am0, const __grid_constant__ CUtensorMap bm0,
       const __grid_constant__ CUtensorMap am1, const __grid_constant__ CUtensorMap bm1) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem0 = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem0 - smem_u32(smem_raw));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_gen + kStages * kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* epi_bar = acc_empty + 2;         // the 128 epilogue threads meet here (bounded waits)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epi_bar + 1);
  uint32_t* last_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nunits = a.total_units;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(epi_bar, 128);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&am0);
    tma_prefetch_desc(&bm0);
    if (a.nprob > 1) {
      tma_prefetch_desc(&am1);
      tma_prefetch_desc(&bm1);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool alive = true;
      for (int u = blockIdx.x; u < nunits && alive; u += gridDim.x) {
        const UnitPos w = unit_pos(a, u);
        const RankProblem& p = a.p[w.prob];
        const CUtensorMap* am = w.prob ? &am1 : &am0;
        const CUtensorMap* bm = w.prob ? &bm1 : &bm0;
        // two consecutive k-steps at a time: both stages are claimed first and
        // their loads issued back to back, so every row of the long operand is
        // requested in 256-byte runs rather than 128-byte ones
        for (int j = 0; j < w.nk && alive; j += 2) {
          const int cnt = w.nk - j < 2 ? w.nk - j : 2;
          for (int q = 0; q < cnt; ++q) {
            const uint32_t stage = (it + q) % kStages, phase = ((it + q) / kStages) & 1u;
            if (!mbar_wait(&empty[stage], phase ^ 1u, a.err)) { alive = false; break; }
          }
          if (!alive) break;
          for (int q = 0; q < cnt; ++q, ++it) {
            const uint32_t stage = it % kStages;
            uint8_t* sA = smem_gen + stage * kStageBytes;
            uint8_t* sB = sA + kABytes;
            const int k0 = (w.kbeg + j + q) * 64;
            mbar_arrive_expect_tx(&full[stage], kStageBytes);
            if (p.a_mn) {   // A^T stored [k][m]: two 64-wide MN boxes
              tma_load_2d(sA, am, w.mt * 128, k0, &full[stage]);
              tma_load_2d(sA + 8192, am, w.mt * 128 + 64, k0, &full[stage]);
            } else {
              tma_load_2d(sA, am, k0, w.mt * 128, &full[stage]);
            }
            if (p.b_mn) tma_load_2d(sB, bm, w.nt * 64, k0, &full[stage]);
            else tma_load_2d(sB, bm, k0, w.nt * 64, &full[stage]);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, uctr = 0;
      bool alive = true;
      for (int u = blockIdx.x; u < nunits && alive; u += gridDim.x, ++uctr) {
        const UnitPos w = unit_pos(a, u);
        const RankProblem& p = a.p[w.prob];
        const uint32_t idesc = idesc_bf16(128, 64, p.a_mn != 0, p.b_mn != 0);
        const uint32_t ab = uctr & 1u, aphase = (uctr >> 1) & 1u;
        if (!mbar_wait(&acc_empty[ab], aphase ^ 1u, a.err)) break;
        tc_fence_after();
        for (int j = 0; j < w.nk; ++j, ++it) {
          const uint32_t stage = it % kStages, phase = (it / kStages) & 1u;
          if (!mbar_wait(&full[stage], phase, a.err)) { alive = false; break; }
          tc_fence_after();
          const uint32_t sA = smem0 + stage * kStageBytes;
          const uint32_t sB = sA + kABytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t adesc = p.a_mn ? smem_desc_sw128(sA + kk * 2048, 8192, 1024)
                                          : smem_desc_sw128(sA + kk * 32, 16, 1024);
            const uint64_t bdesc = p.b_mn ? smem_desc_sw128(sB + kk * 2048, 8192, 1024)
                                          : smem_desc_sw128(sB + kk * 32, 16, 1024);
            mma_bf16_ss(tmem_base + ab * 64, adesc, bdesc, idesc, (j | kk) != 0 ? 1u : 0u);
          }
          mma_commit(&empty[stage]);
        }
        if (alive) mma_commit(&acc_full[ab]);
      }
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int quarter = warp & 3;            // warps 2,3,4,5 -> TMEM lane quarters 2,3,0,1
    const int et = (warp - 2) * 32 + lane;   // 0 .. 127
    uint32_t uctr = 0, ephase = 0;
    // all 128 epilogue threads arrive, then wait for the phase (bounded)
    auto epi_sync = [&]() -> bool {
      mbar_arrive(epi_bar);
      const bool ok = mbar_wait(epi_bar, ephase, a.err);
      ephase ^= 1u;
      return ok;
    };
    for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++uctr) {
      const UnitPos w = unit_pos(a, u);
      const RankProblem& p = a.p[w.prob];
      const uint32_t ab = uctr & 1u, aphase = (uctr >> 1) & 1u;
      if (!mbar_wait(&acc_full[ab], aphase, a.err)) break;
      tc_fence_after();
      const int rl = quarter * 32 + lane;                   // row inside the tile
      const int64_t row = static_cast<int64_t>(w.mt) * 128 + rl;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + ab * 64;
      float v[64];
      {
        uint32_t r0[32], r1[32];
        tmem_ld32(taddr, r0);
        tmem_ld32(taddr + 32, r1);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          v[c] = __uint_as_float(r0[c]);
          v[32 + c] = __uint_as_float(r1[c]);
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);                           // TMEM free for the next unit
      const int64_t c0 = static_cast<int64_t>(w.nt) * 64;
      if (p.splits == 1) {
        store_final(p, row, c0, v);
        continue;
      }
      // split contraction: partial to this split's slot ([64 cols][128 rows],
      // coalesced per column), then count; the unit completing the count sums
      // all slots of the tile in split order
      const int tile = w.mt * p.n_tiles + w.nt;
      float* slot_tile = p.slots + static_cast<int64_t>(tile) * p.splits * (64 * 128);
      float* mine = slot_tile + static_cast<int64_t>(w.sp) * (64 * 128);
#pragma unroll
      for (int c = 0; c < 64; ++c) mine[c * 128 + rl] = v[c];
      __threadfence();
      if (!epi_sync()) break;
      if (et == 0) *last_flag = (atomicAdd(p.counters + tile, 1u) == static_cast<uint32_t>(p.splits - 1)) ? 1u : 0u;
      if (!epi_sync()) break;
      const bool last = *last_flag != 0u;
      if (!last) continue;
      __threadfence();
      float sum[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) sum[c] = 0.0f;
      for (int s = 0; s < p.splits; ++s) {
        if (s == w.sp) {
#pragma unroll
          for (int c = 0; c < 64; ++c) sum[c] += v[c];
        } else {
          const float* src = slot_tile + static_cast<int64_t>(s) * (64 * 128) + rl;
#pragma unroll
          for (int c = 0; c < 64; ++c) sum[c] += __ldcg(src + c * 128);
        }
      }
      store_final(p, row, c0, sum);
    }
    // side job: bf16(scale * in) of a caller's fp32 matrix, zero-padded,
    // one row per epilogue thread over the whole grid
    if (a.cvt_in) {
      const int64_t gt = static_cast<int64_t>(blockIdx.x) * 128 + et;
      for (int64_t i = gt; i < a.cvt_rows; i += static_cast<int64_t>(gridDim.x) * 128) {
        const float* src = a.cvt_in + i * a.cvt_ld_in;
        uint16_t* dst = a.cvt_out + i * a.cvt_ld_out;
        for (int64_t c = 0; c < a.cvt_cols_out; c += 8) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = (c + e < a.cvt_cols) ? __fmul_rn(a.cvt_scale, src[c + e]) : 0.0f;
          uint4 q;
          q.x = pack_bf16x2(f[0], f[1]);
          q.y = pack_bf16x2(f[2], f[3]);
          q.z = pack_bf16x2(f[4], f[5]);
          q.w = pack_bf16x2(f[6], f[7]);
          *reinterpret_cast<uint4*>(dst + c) = q;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

std::atomic<uint64_t> g_attr_done{0};

}  // namespace

int rank_splits(int tiles, int ksteps, int num_sms, int max_splits) {
  // makespan model: waves of units over the SMs times the k-steps of a unit
  // plus two k-steps of fixed cost (epilogue, split fix-up)
  // each split adds a 32 KB partial tile written and read back: beyond the
  // splits a tile needs to spread over the SMs (about two units per SM), at
  // most 4
  int spread = tiles > 0 ? (2 * num_sms + tiles - 1) / tiles : 1;
  if (spread < 4) spread = 4;
  if (max_splits > spread) max_splits = spread;
  int best = 1;
  int64_t best_cost = -1;
  const int cap = ksteps / 4 > 1 ? ksteps / 4 : 1;          // at least 4 k-steps per split
  for (int s = 1; s <= max_splits && s <= cap; ++s) {
    const int64_t waves = (static_cast<int64_t>(tiles) * s + num_sms - 1) / num_sms;
    const int64_t cost = waves * ((ksteps + s - 1) / s + 2);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

size_t rank_slot_bytes(int tiles, int splits) {
  return splits > 1 ? static_cast<size_t>(tiles) * splits * 64 * 128 * sizeof(float) : 0;
}

cudaError_t launch_rank(const RankArgs& args, const CUtensorMap& am0, const CUtensorMap& bm0,
                        const CUtensorMap& am1, const CUtensorMap& bm1, int num_sms, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(g_attr_done.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(k_rank, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmem));
    if (e != cudaSuccess) return e;
    g_attr_done.fetch_or(bit, std::memory_order_acq_rel);
  }
  const int grid = args.total_units < num_sms ? args.total_units : num_sms;
  k_rank<<<grid, kThreads, kSmem, stream>>>(args, am0, bm0, am1, bm1);
  return cudaGetLastError();
}

}  // namespace qlora
