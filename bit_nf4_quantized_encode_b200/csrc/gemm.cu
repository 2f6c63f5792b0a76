// gemm.cu -- tcgen05 / TMEM / TMA GEMM kernels for sm_100a.
//
// What is computed (QLoRA, arXiv:2305.14314; automatone "QLoRA paper
// explained", section "How it works": the frozen 4-bit weight is dequantized to
// bf16 on the fly for the forward and backward matmuls, and gradients land only
// on the 16-bit LoRA adapters):
//   forward    Y  = X deq(W)^T + s (X A^T) B^T
//   backward   dX = dY deq(W) + s (dY B) A,  dB = s dY^T (X A^T),  dA = s (dY B)^T X
//
// Orientation: the fused kernel computes D^T, i.e. D[rows of the weight side,
// tokens] so that the dequantized weight tile is the 128-row MMA operand A
// (written to shared memory by dequant warps) and the activation tile is the
// N operand (TMA).  Each expanded weight element then serves a 256-token tile.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "gemm.h"
#include "nf4_device.cuh"
#include "sm100_ptx.cuh"

namespace qlora {

namespace {

constexpr int kATileBytes = 128 * 128;     // 128 rows x 64 bf16, 128B-swizzled
constexpr int kDequantGroups = 4;          // groups of 128 threads; group g takes k-steps = g mod 4
constexpr int kNumDequantWarps = 4 * kDequantGroups;
constexpr int kEpiWarp0 = kNumDequantWarps;          // 4 epilogue warps (TMEM lane quarters 0..3)
constexpr int kTmaWarp = kEpiWarp0 + 4;
constexpr int kMmaWarp = kTmaWarp + 1;
constexpr int kFusedThreads = (kMmaWarp + 1) * 32;

__host__ __device__ constexpr int fused_stages(int bn) { return bn >= 128 ? 4 : 8; }
static_assert(kDequantGroups == 4, "stage ring and group rotation assume four groups");
__host__ __device__ constexpr int fused_tmem_cols(int bn) { return 2 * bn < 32 ? 32 : 2 * bn; }
// Packed codes of one dequant task set (4 KB: 128 rows x 32 B forward, 64 rows
// x 64 B backward), loaded by TMA into one of two slots per dequant group.
constexpr int kCodeSlotBytes = 4096;
constexpr int kCodeSlots = 2 * kDequantGroups;
__host__ __device__ constexpr size_t fused_smem_bytes(int bn) {
  return 1024 + static_cast<size_t>(fused_stages(bn)) * (kATileBytes + bn * 128) +
         static_cast<size_t>(kCodeSlots) * kCodeSlotBytes + 512;
}

// Work unit -> (m-tile, token tile, split) and its k-step range.  Units run in
// groups of m_group m-tiles: inside a group the m-tile varies fastest (after the
// split) and the group sweeps every token tile before the next group starts, so
// the codes of one group (a few tens of MB) stay in L2 while every token tile
// re-reads them, and a token tile of activations is reused by the whole group.
struct Unit {
  int mt, tt, sp;
  int kbeg, kmain;     // first main k-step, number of main k-steps
  int nk;              // main + LoRA k-steps
};

__device__ __forceinline__ Unit decode_unit(int u, int m_tiles, int t_tiles, int m_group, int splits,
                                            int ksteps, int lora_steps) {
  Unit w;
  w.sp = u % splits;
  const int rest = u / splits;
  const int per_group = m_group * t_tiles;
  const int gi = rest / per_group;
  const int r2 = rest - gi * per_group;
  const int gsz = min(m_group, m_tiles - gi * m_group);      // the last group may be short
  w.mt = gi * m_group + r2 % gsz;
  w.tt = r2 / gsz;
  w.kbeg = static_cast<int>((static_cast<int64_t>(ksteps) * w.sp) / splits);
  const int kend = static_cast<int>((static_cast<int64_t>(ksteps) * (w.sp + 1)) / splits);
  w.kmain = kend - w.kbeg;
  w.nk = w.kmain + (w.sp == 0 ? lora_steps : 0);
  return w;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w) : "memory");
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr) : "memory");
  return v;
}

// Prefetched inputs of one dequant task.
struct DqLoad {
  uint4 c0, c1;        // 64 packed codes (32 bytes)
  uint32_t q;          // E4M3 block constant
  float c2;            // second-level absmax of its group (without double quantization: c1 itself)
  bool valid;
};

// The task's block constant and c2 (its 32 code bytes arrive by TMA: with a
// load per thread, one L2 request per row, the kernel ran 4-5% slower).
template <int kDir>
__device__ __forceinline__ DqLoad dq_load(const FusedArgs& a, int m0, int kstep, int t) {
  DqLoad d;
  int64_t n, kcol;
  if (kDir == 0) {              // forward: task = W row m0 + t, block kstep
    n = m0 + t;
    kcol = static_cast<int64_t>(kstep) * 64;
  } else {                      // backward: task = W row kstep*64 + t/2, cols m0 + 64*(t&1)
    n = static_cast<int64_t>(kstep) * 64 + (t >> 1);
    kcol = m0 + 64 * (t & 1);
  }
  d.valid = (n < a.nw) && (kcol < a.kw);
  if (d.valid) {
    const int64_t e = n * a.kw + kcol;                 // first weight of the block
    const int64_t blk = e >> 6;
    if (a.absf) {                 // no double quantization: the constant itself
      d.q = 0;
      d.c2 = __ldg(a.absf + blk);
    } else {
      d.q = __ldg(a.qabs + blk);
      d.c2 = __ldg(a.c2 + (blk >> 8));
    }
  }
  return d;
}

// Byte offset of this task's 128-byte row inside the A tile.
template <int kDir>
__device__ __forceinline__ uint32_t task_row_base(int t, uint32_t& swz_row) {
  if (kDir == 0) { swz_row = t; return static_cast<uint32_t>(t) * 128u; }
  swz_row = t >> 1;                               // K-row inside the MN-major tile
  return static_cast<uint32_t>(t & 1) * 8192u + static_cast<uint32_t>(t >> 1) * 128u;
}

template <int kDir>
__device__ __forceinline__ void dq_store(uint32_t sA, int t, const DqLoad& d, float mu, bool plain,
                                         const CodebookParam& cb) {
  uint32_t r;
  const uint32_t base = sA + task_row_base<kDir>(t, r);
  if (!d.valid) {
    const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int c = 0; c < 8; ++c) st_shared_v4(base + (((c ^ (r & 7)) << 4)), z);
    return;
  }
  const float c1p = plain ? d.c2 : block_constant(d.q, __fdiv_rn(d.c2, 448.0f), mu);
  const ByteTables tb = make_tables(cb.level, c1p);
  const uint32_t w[8] = {d.c0.x, d.c0.y, d.c0.z, d.c0.w, d.c1.x, d.c1.y, d.c1.z, d.c1.w};
#pragma unroll
  for (int c = 0; c < 8; ++c) st_shared_v4(base + (((c ^ (r & 7)) << 4)), expand8(w[c], tb));
}

// The LoRA weight rows for the appended k-steps: a plain copy into the same
// swizzled layout (forward: B rows, K-major over r; backward: A rows, MN-major).
template <int kDir>
__device__ __forceinline__ void lora_store(const FusedArgs& a, uint32_t sA, int m0, int rs, int t) {
  uint32_t r;
  const uint32_t base = sA + task_row_base<kDir>(t, r);
  const uint16_t* src = nullptr;
  int nvalid = 0;  // valid 8-element chunks
  if (kDir == 0) {
    const int64_t n = m0 + t;
    const int r0 = rs * 64;
    if (n < a.nw) {
      src = a.lora_w + n * a.r + r0;
      nvalid = min(64, a.r - r0) / 8;
    }
  } else {
    const int ridx = rs * 64 + (t >> 1);
    const int64_t kcol = m0 + 64 * (t & 1);
    if (ridx < a.r && kcol < a.kw) {
      src = a.lora_w + static_cast<int64_t>(ridx) * a.kw + kcol;
      nvalid = 8;
    }
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint4 v = make_uint4(0, 0, 0, 0);
    if (c < nvalid) v = __ldg(reinterpret_cast<const uint4*>(src) + c);
    st_shared_v4(base + (((c ^ (r & 7)) << 4)), v);
  }
}

template <int kDir, int kBN>
__global__ void __launch_bounds__(kFusedThreads, 1)
k_fused(const FusedArgs a, const __grid_constant__ CUtensorMap act,
        const __grid_constant__ CUtensorMap lora_act, const __grid_constant__ CUtensorMap codes_map) {
  constexpr int kStages = fused_stages(kBN);
  constexpr int kBTileBytes = kBN * 128;
  constexpr int kStageBytes = kATileBytes + kBTileBytes;
  constexpr uint32_t kTmemCols = fused_tmem_cols(kBN);
  constexpr uint32_t kIdesc = idesc_bf16(128, kBN, kDir == 1, false);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t smem0 = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem0 - smem_u32(smem_raw));
  const uint32_t code0 = smem0 + kStages * kStageBytes;     // kCodeSlots code slots
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_gen + kStages * kStageBytes + kCodeSlots * kCodeSlotBytes);
  uint64_t* full_a = bars;                   // [kStages] dequant -> MMA (128 arrivals)
  uint64_t* full_b = bars + kStages;         // [kStages] TMA -> MMA (tx bytes)
  uint64_t* empty = bars + 2 * kStages;      // [kStages] MMA -> producers (commit)
  uint64_t* acc_full = bars + 3 * kStages;   // [2] MMA -> epilogue (commit)
  uint64_t* acc_empty = acc_full + 2;        // [2] epilogue -> MMA (128 arrivals)
  uint64_t* code_full = acc_empty + 2;       // [kCodeSlots] code TMA -> dequant group (tx bytes)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(code_full + kCodeSlots);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nunits = a.m_tiles * a.t_tiles * a.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_a[s], 128);
      mbar_init(&full_b[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    for (int c = 0; c < kCodeSlots; ++c) mbar_init(&code_full[c], 1);
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kTmaWarp && lane == 0) {
    tma_prefetch_desc(&act);
    tma_prefetch_desc(&lora_act);
    tma_prefetch_desc(&codes_map);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < kNumDequantWarps) {
    // ------------------------------------------------ dequant producers
    const int group = warp >> 2;              // warps 4g .. 4g+3
    const int t = threadIdx.x & 127;
    const bool plain = a.absf != nullptr;
    const float mu = plain ? 0.0f : __ldg(a.mean);
    // The group's code tiles come by TMA into two slots, one task ahead.  A
    // slot is refilled only after this thread's wait on `empty` for the current
    // task, which implies every thread of the group has finished the task
    // before it, the last reader of that slot.
    uint32_t ci = 0;                          // code tasks of this group so far
    auto issue_codes = [&](uint32_t c, int m0, int kstep) {
      const int slot = group * 2 + static_cast<int>(c & 1u);
      mbar_arrive_expect_tx(&code_full[slot], kCodeSlotBytes);
      uint8_t* dst = smem_gen + kStages * kStageBytes + slot * kCodeSlotBytes;
      if (kDir == 0) tma_load_2d(dst, &codes_map, kstep * 32, m0, &code_full[slot]);
      else tma_load_2d(dst, &codes_map, m0 / 2, kstep * 64, &code_full[slot]);
    };
    uint32_t gctr = 0;
    bool alive = true;
    for (int u = blockIdx.x; u < nunits && alive; u += gridDim.x) {
      const Unit w = decode_unit(u, a.m_tiles, a.t_tiles, a.m_group, a.splits, a.ksteps, a.lora_steps);
      const int m0 = w.mt * 128;
      int j = static_cast<int>((static_cast<uint32_t>(group) - gctr) & (kDequantGroups - 1));
      DqLoad next;
      if (j < w.kmain) {
        next = dq_load<kDir>(a, m0, w.kbeg + j, t);
        if (t == 0) issue_codes(ci, m0, w.kbeg + j);
      }
      for (; j < w.nk; j += kDequantGroups) {
        const uint32_t it = gctr + j;
        const uint32_t stage = it % kStages, phase = (it / kStages) & 1u;
        DqLoad cur = next;
        if (j + kDequantGroups < w.kmain) next = dq_load<kDir>(a, m0, w.kbeg + j + kDequantGroups, t);
        if (!mbar_wait(&empty[stage], phase ^ 1u, a.err)) { alive = false; break; }
        if (t == 0 && j + kDequantGroups < w.kmain) issue_codes(ci + 1, m0, w.kbeg + j + kDequantGroups);
        const uint32_t sA = smem0 + stage * kStageBytes;
        if (j < w.kmain) {
          const int slot = group * 2 + static_cast<int>(ci & 1u);
          if (!mbar_wait(&code_full[slot], (ci >> 1) & 1u, a.err)) { alive = false; break; }
          const uint32_t src = code0 + slot * kCodeSlotBytes + static_cast<uint32_t>(t) * 32u;
          cur.c0 = lds_v4(src);
          cur.c1 = lds_v4(src + 16);
          ++ci;
          dq_store<kDir>(sA, t, cur, mu, plain, a.cb);
        } else {
          lora_store<kDir>(a, sA, m0, j - w.kmain, t);
        }
        fence_proxy_async_smem();
        mbar_arrive(&full_a[stage]);
      }
      gctr += w.nk;
    }
  } else if (warp == kTmaWarp) {
    // ------------------------------------------------ TMA producer (activations)
    if (lane == 0) {
      uint32_t gctr = 0;
      bool alive = true;
      for (int u = blockIdx.x; u < nunits && alive; u += gridDim.x) {
        const Unit w = decode_unit(u, a.m_tiles, a.t_tiles, a.m_group, a.splits, a.ksteps, a.lora_steps);
        for (int j = 0; j < w.nk; ++j) {
          const uint32_t it = gctr + j;
          const uint32_t stage = it % kStages, phase = (it / kStages) & 1u;
          if (!mbar_wait(&empty[stage], phase ^ 1u, a.err)) { alive = false; break; }
          uint8_t* sB = smem_gen + stage * kStageBytes + kATileBytes;
          mbar_arrive_expect_tx(&full_b[stage], kBTileBytes);
          if (j < w.kmain)
            tma_load_2d(sB, &act, (w.kbeg + j) * 64, w.tt * kBN, &full_b[stage]);
          else
            tma_load_2d(sB, &lora_act, (j - w.kmain) * 64, w.tt * kBN, &full_b[stage]);
        }
        gctr += w.nk;
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t gctr = 0, uctr = 0;
      bool alive = true;
      for (int u = blockIdx.x; u < nunits && alive; u += gridDim.x, ++uctr) {
        const Unit w = decode_unit(u, a.m_tiles, a.t_tiles, a.m_group, a.splits, a.ksteps, a.lora_steps);
        const uint32_t ab = uctr & 1u, aphase = (uctr >> 1) & 1u;
        if (!mbar_wait(&acc_empty[ab], aphase ^ 1u, a.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * kBN;
        for (int j = 0; j < w.nk; ++j) {
          const uint32_t it = gctr + j;
          const uint32_t stage = it % kStages, phase = (it / kStages) & 1u;
          if (!mbar_wait(&full_a[stage], phase, a.err) || !mbar_wait(&full_b[stage], phase, a.err)) {
            alive = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem0 + stage * kStageBytes;
          const uint32_t sB = sA + kATileBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t adesc = (kDir == 0) ? smem_desc_sw128(sA + kk * 32, 16, 1024)
                                               : smem_desc_sw128(sA + kk * 2048, 8192, 1024);
            const uint64_t bdesc = smem_desc_sw128(sB + kk * 32, 16, 1024);
            mma_bf16_ss(d_tmem, adesc, bdesc, kIdesc, (j | kk) != 0 ? 1u : 0u);
          }
          mma_commit(&empty[stage]);
        }
        if (alive) mma_commit(&acc_full[ab]);
        gctr += w.nk;
      }
    }
  } else {
    // ------------------------------------------------ epilogue: TMEM -> global
    const int quarter = warp & 3;             // the four epilogue warps cover lane quarters 0..3
    uint32_t uctr = 0;
    for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++uctr) {
      const Unit w = decode_unit(u, a.m_tiles, a.t_tiles, a.m_group, a.splits, a.ksteps, a.lora_steps);
      const uint32_t ab = uctr & 1u, aphase = (uctr >> 1) & 1u;
      if (!mbar_wait(&acc_full[ab], aphase, a.err)) break;
      tc_fence_after();
      const int64_t row = static_cast<int64_t>(w.mt) * 128 + quarter * 32 + lane;
      const bool row_ok = row < a.mdim;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + ab * kBN;
#pragma unroll 1
      for (int cc = 0; cc < kBN / 32 || (kBN < 32 && cc == 0); ++cc) {
        uint32_t v[32];
        if constexpr (kBN >= 32) {
          tmem_ld32(taddr + cc * 32, v);
        } else {
          uint32_t v16[16];
          tmem_ld16(taddr, v16);
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = v16[i];
        }
        tmem_wait_ld();
        constexpr int kCols = kBN < 32 ? kBN : 32;
#pragma unroll
        for (int c = 0; c < kCols; ++c) {
          const int64_t tok = static_cast<int64_t>(w.tt) * kBN + cc * 32 + c;
          if (row_ok && tok < a.m) {
            const float val = __uint_as_float(v[c]);
            if (a.splits > 1) {
              atomicAdd(a.out_acc + tok * a.ldo + row, val);
            } else {
              const __nv_bfloat16 b = __float2bfloat16_rn(val);
              __stcs(a.out + tok * a.ldo + row, *reinterpret_cast<const unsigned short*>(&b));   // streamed out
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------------------ converts
__device__ __forceinline__ void store_out(uint16_t* p, float v) {
  const __nv_bfloat16 b = __float2bfloat16_rn(v);
  *p = *reinterpret_cast<const uint16_t*>(&b);
}

template <typename T>
__global__ void k_convert(const float* __restrict__ in, int64_t rows, int64_t cols_in, int64_t ld_in,
                          int64_t cols_out, float scale, T* __restrict__ out, int64_t ld_out) {
  const int64_t n = rows * cols_out;
  for (int64_t o = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; o < n;
       o += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = o / cols_out, j = o % cols_out;
    const float v = j < cols_in ? __fmul_rn(in[i * ld_in + j], scale) : 0.0f;
    store_out(out + i * ld_out + j, v);
  }
}

// ------------------------------------------------------------------ few-token LoRA gradients
// One thread per output element; M <= 16 terms each, fp32 accumulation in
// token order.  dA threads walk k (coalesced X reads and dA writes, G[m, j]
// uniform across a warp); dB threads walk j (coalesced XA reads and dB
// writes, dY[m, n] uniform across the 64-wide j run).
__global__ void k_small_grads(const float* __restrict__ G, int64_t ld_g, const float* __restrict__ XA,
                              int64_t ld_xa, const uint16_t* __restrict__ X,
                              const uint16_t* __restrict__ dY, int64_t M, int64_t rows, int64_t cols,
                              int r, float s, float* __restrict__ dA, float* __restrict__ dB) {
  const int64_t na = static_cast<int64_t>(r) * cols;
  const int64_t nb = rows * r;
  for (int64_t o = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; o < na + nb;
       o += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float acc = 0.0f;
    if (o < na) {
      const int64_t j = o / cols, k = o % cols;
      for (int64_t m = 0; m < M; ++m)
        acc = __fmaf_rn(G[m * ld_g + j], bf16_lo(X[m * cols + k]), acc);
      dA[o] = __fmul_rn(acc, s);
    } else {
      const int64_t q = o - na;
      const int64_t n = q / r, j = q % r;
      for (int64_t m = 0; m < M; ++m)
        acc = __fmaf_rn(bf16_lo(dY[m * rows + n]), XA[m * ld_xa + j], acc);
      dB[q] = __fmul_rn(acc, s);
    }
  }
}

int grid_for(int64_t n, int num_sms) {
  const int64_t want = (n + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  return static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
}

// Raises a kernel's dynamic shared-memory limit once per device (not inside
// every launch, so launches stay legal during CUDA-graph capture).
template <typename K>
cudaError_t ensure_smem_attr(K kernel, size_t bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

template <int kDir, int kBN>
cudaError_t launch_fused_t(const FusedArgs& args, const CUtensorMap& act, const CUtensorMap& lora_act,
                           const CUtensorMap& codes_map, int num_sms, cudaStream_t stream) {
  static std::atomic<uint64_t> attr_done{0};
  const size_t smem = fused_smem_bytes(kBN);
  cudaError_t e = ensure_smem_attr(k_fused<kDir, kBN>, smem, attr_done);
  if (e != cudaSuccess) return e;
  const int nunits = args.m_tiles * args.t_tiles * args.splits;
  const int grid = nunits < num_sms ? nunits : num_sms;
  k_fused<kDir, kBN><<<grid, kFusedThreads, smem, stream>>>(args, act, lora_act, codes_map);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fused(FusedDir dir, int token_tile, const FusedArgs& args, const CUtensorMap& act,
                         const CUtensorMap& lora_act, const CUtensorMap& codes_map, int num_sms,
                         cudaStream_t stream) {
  if (dir == FusedDir::kFwd) {
    // the decode-shaped forward (16 tokens or fewer) is k_gemv's
    if (token_tile == 256) return launch_fused_t<0, 256>(args, act, lora_act, codes_map, num_sms, stream);
  } else {
    if (token_tile == 256) return launch_fused_t<1, 256>(args, act, lora_act, codes_map, num_sms, stream);
    if (token_tile == 16) return launch_fused_t<1, 16>(args, act, lora_act, codes_map, num_sms, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_convert_bf16(const float* in, int64_t rows, int64_t cols_in, int64_t ld_in,
                                int64_t cols_out, float scale, uint16_t* out, int64_t ld_out, int num_sms,
                                cudaStream_t stream) {
  const int64_t n = rows * cols_out;
  if (n == 0) return cudaSuccess;
  k_convert<uint16_t><<<grid_for(n, num_sms), 256, 0, stream>>>(in, rows, cols_in, ld_in, cols_out, scale,
                                                             out, ld_out);
  return cudaGetLastError();
}

cudaError_t launch_small_grads(const float* G, int64_t ld_g, const float* XA, int64_t ld_xa,
                               const uint16_t* X, const uint16_t* dY, int64_t M, int64_t rows,
                               int64_t cols, int r, float s, float* dA, float* dB, int num_sms,
                               cudaStream_t stream) {
  const int64_t n = static_cast<int64_t>(r) * (cols + rows);
  k_small_grads<<<grid_for(n, num_sms), 256, 0, stream>>>(G, ld_g, XA, ld_xa, X, dY, M, rows, cols, r, s,
                                                      dA, dB);
  return cudaGetLastError();
}

}  // namespace qlora
