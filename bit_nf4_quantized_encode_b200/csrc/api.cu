// api.cu -- the C ABI of libqlora (declared in include/qlora.h): argument
// validation, work-buffer layout, TMA descriptors and the launch sequences of
// quantize, dequantize, forward and backward.  Every step of the hot path runs
// in the kernels of codec.cu and gemm.cu; this file only marshals arguments.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <atomic>
#include <cstring>
#include <mutex>

#include "codec.h"
#include "gemm.h"
#include "gemv.h"
#include "internal.h"
#include "lora.h"
#include "nf4_tables.h"
#include "qlora.h"

namespace qlora {

__device__ uint32_t g_device_errors;   // bit flags written by kernels (see sm100_ptx.cuh)

namespace {

constexpr int kBlock = 64;
constexpr int kBlock2 = 256;
constexpr int kMaxEncodeGrid = 2048;        // partial sums of the mean: one double per CTA
constexpr int64_t kMaxDim = int64_t(1) << 31;
constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  bool sm100 = false;
  int num_sms = 0;
  uint32_t* err = nullptr;
};

std::mutex g_mu;
std::atomic<uint64_t> g_launches{0};
thread_local cudaEvent_t t_gemm_start = nullptr, t_gemm_stop = nullptr;

bool make_map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch_bytes,
                 uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz);

cudaError_t fused_timed(FusedDir dir, int bn, const FusedArgs& fa, const CUtensorMap& act,
                        const CUtensorMap& lora, int num_sms, cudaStream_t cs) {
  // the dequant groups' code tiles: forward 128 rows x 32 bytes (one block of
  // each row), backward 64 rows x 64 bytes (two blocks of each row)
  CUtensorMap codes_map;
  const bool fwd = dir == FusedDir::kFwd;
  if (!make_map_u8(&codes_map, fa.codes, static_cast<uint64_t>(fa.kw / 2), static_cast<uint64_t>(fa.nw),
                   static_cast<uint64_t>(fa.kw / 2), fwd ? 32 : 64, fwd ? 128 : 64, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  cudaEvent_t e0 = t_gemm_start, e1 = t_gemm_stop;
  t_gemm_start = t_gemm_stop = nullptr;
  if (e0 && cudaEventRecord(e0, cs) != cudaSuccess) return cudaErrorUnknown;
  cudaError_t e = counted(launch_fused(dir, bn, fa, act, lora, codes_map, num_sms, cs));
  if (e == cudaSuccess && e1) e = cudaEventRecord(e1, cs);
  return e;
}
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;

qlora_status device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QLORA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return QLORA_ERR_CUDA;
    d.sm100 = (major == 10 && minor == 0);
    d.num_sms = sms;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_errors) != cudaSuccess) return QLORA_ERR_CUDA;
    d.err = static_cast<uint32_t*>(p);
    if (!g_encode_tiled) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr)
        return QLORA_ERR_CUDA;
      g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    d.ready = true;
  }
  if (!d.sm100) return QLORA_ERR_UNSUPPORTED;
  *out = d;
  return QLORA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// 2-D bf16 tensor map, 128-byte swizzle: dims {inner, outer}, row pitch in
// bytes, box {64, box_outer}.  Out-of-bounds elements read as zero.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch_bytes,
              uint32_t box_outer) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch_bytes};
  const cuuint32_t box[2] = {64, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
                                    dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D uint8 tensor map without swizzle (packed NF4 codes): dims {inner, outer}.
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch_bytes,
                 uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// m-tiles per rasterization group of the fused kernel: the packed codes of one
// group (128 rows or columns of W times `contraction` weights, half a byte
// each) should take about 48 MB, so that they stay in the 126 MB L2 while the
// group sweeps the token tiles.
int m_group_for(int m_tiles, int64_t contraction) {
  const int64_t per_tile = 64 * contraction;
  int64_t g = (int64_t{48} << 20) / (per_tile > 0 ? per_tile : 1);
  if (g < 1) g = 1;
  if (g > m_tiles) g = m_tiles;
  return static_cast<int>(g);
}

// Split count for `tiles` output tiles of `ksteps` steps each over `sms` CTAs:
// minimises the makespan ceil(tiles * s / sms) * ceil(ksteps / s), counting two
// steps of fixed cost per work unit.
int balanced_splits(int tiles, int ksteps, int sms) {
  int best = 1;
  int64_t best_cost = -1;
  for (int s = 1; s <= ksteps && s <= 128; ++s) {
    const int64_t waves = (static_cast<int64_t>(tiles) * s + sms - 1) / sms;
    const int64_t cost = waves * ((ksteps + s - 1) / s + 2);
    if (best_cost < 0 || cost < best_cost) { best_cost = cost; best = s; }
  }
  return best;
}

CodebookParam codebook_param(int type) {
  CodebookParam cb;
  const Nf4Tables& t = level_tables(type);
  for (int i = 0; i < 16; ++i) cb.level[i] = t.level[i];
  return cb;
}

// fp32 block constants of a weight stored without double quantization, else NULL
const float* plain_absmax(const qlora_nf4_tensor* t) { return t->blocksize2 == 0 ? t->absmax : nullptr; }

qlora_status cuda_status(cudaError_t e) { return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA; }

// ------------------------------------------------------------------ linear layout
struct LinearShape {
  int64_t rows, cols, m;
  int r, rpad, lora_steps;
  bool decode;      // M <= 16: token tile 16, split-K
};

qlora_status check_linear(const qlora_nf4_tensor* W, int64_t M, int32_t r, LinearShape* sh) {
  qlora_status st = check_tensor(W);
  if (st != QLORA_OK) return st;
  if (M < 1 || M > kMaxDim) return QLORA_ERR_SHAPE;
  if (W->rows < 8 || W->cols < 64 || W->cols % 64 != 0 || W->rows % 8 != 0) return QLORA_ERR_SHAPE;
  if (r < 8 || r > 256 || r % 8 != 0) return QLORA_ERR_SHAPE;
  sh->rows = W->rows;
  sh->cols = W->cols;
  sh->m = M;
  sh->r = r;
  sh->lora_steps = (r + 63) / 64;
  sh->rpad = 64 * sh->lora_steps;
  sh->decode = M <= 16;
  return QLORA_OK;
}

// Work buffer layout: fp32 accumulators first (one memset clears them all),
// then bf16 staging.  Offsets in bytes, each 256-aligned.
// The work buffer's split slots are sized independently of the device (for up
// to this many SMs); a launch picks its own split count within that space.
constexpr int kSizingSms = 256;
constexpr int kMaxRankSplits = 32;

// One rank-r contraction's tiling: tiles of 128 rows x 64 columns, K splits.
struct RankPlan {
  int m_tiles, n_tiles, ksteps, splits;
  int tiles() const { return m_tiles * n_tiles; }
};
RankPlan rank_tiling(int64_t mdim, int64_t contraction, int lora_steps) {
  RankPlan p;
  p.m_tiles = static_cast<int>((mdim + 127) / 128);
  p.n_tiles = lora_steps;
  p.ksteps = static_cast<int>((contraction + 63) / 64);
  p.splits = 1;
  return p;
}
// Splits of a launch with `tiles` tiles in all (the problems of one launch
// share them) and `ksteps` k-steps, within `slot_bytes` of slot space.
int launch_splits(int tiles, int ksteps, int num_sms, size_t slot_bytes) {
  // a split count s > 1 needs tiles * s partial tiles of slot space
  const size_t per_split = static_cast<size_t>(tiles) * 64 * 128 * sizeof(float);
  size_t cap = kMaxRankSplits;
  if (per_split > 0 && slot_bytes / per_split < cap) cap = slot_bytes / per_split;
  return rank_splits(tiles, ksteps, num_sms, cap < 2 ? 1 : static_cast<int>(cap));
}
// The plan of a launch must fit its slot region; checked before every launch.
bool slots_fit(int tiles, int splits, size_t slot_bytes) {
  return rank_slot_bytes(tiles, splits) <= slot_bytes;
}
// Slot space of a launch: the most any of these SM counts plans for, so a
// buffer sized without a device lets the launch use its own best split count.
size_t sized_slots(int tiles, int ksteps) {
  static const int kSmCounts[] = {96, 108, 114, 120, 128, 132, 144, 148, 152, 160, 170, 188, 192, 224, kSizingSms};
  size_t most = 0;
  for (int sms : kSmCounts) {
    const size_t b = rank_slot_bytes(tiles, rank_splits(tiles, ksteps, sms, kMaxRankSplits));
    if (b > most) most = b;
  }
  return most;
}

// Work buffer layout: the region cleared by one memset first (counters, and
// the decode backward's split-K dX accumulator), then the rest.  Offsets in
// bytes, each 256-aligned; every size is independent of the device.
struct FwdLayout {
  size_t cnt, slots, xa_slices, sxa, rank_cnt, rank_slots, rank_slot_bytes, clear_end, total;
};
FwdLayout fwd_layout(const LinearShape& s) {
  FwdLayout l{};
  size_t o = 0;
  if (s.decode) {        // k_xa_zero + k_gemv: tile counters, partial slots, X A^T slices
    const size_t m_tiles = (size_t(s.rows) + gemv_tile_rows() - 1) / gemv_tile_rows();
    const size_t steps = (size_t(s.cols) / 64 + 3) / 4;
    l.cnt = o;      o = round_up(o + m_tiles * 8 * 4, 256);
    l.slots = o;    o = round_up(o + size_t(gemv_slot_floats(int64_t(m_tiles), int64_t(steps))) * 4, 256);
    l.xa_slices = o; o = round_up(o + size_t(kMaxXaSplits) * 16 * s.rpad * 4, 256);
    l.clear_end = 0;
    l.total = o;
    return l;
  }
  // k_rank (X A^T -> bf16(s X A^T)) then the fused dequant-GEMM
  const RankPlan xa = rank_tiling(s.m, s.cols, s.lora_steps);
  l.rank_cnt = o;   o = round_up(o + size_t(xa.tiles()) * 4, 256);
  l.clear_end = o;
  l.rank_slot_bytes = sized_slots(xa.tiles(), xa.ksteps);
  l.rank_slots = o; o = round_up(o + l.rank_slot_bytes, 256);
  l.sxa = o;        o = round_up(o + size_t(s.m) * s.rpad * 2, 256);
  l.total = o;
  return l;
}

// Backward: launch 1 = dY B (and X A^T when it is not supplied), launch 2 =
// the fused dX, launch 3 = dY^T (s X A^T) and X^T (s dY B) (more than 16
// tokens; with fewer, k_small_grads from the fp32 G and X A^T).  Launch 1's
// slot space covers both of its forms.
struct BwdLayout {
  size_t cnt1, cnt2, dx_acc, clear_end, slots1, slots1_bytes, slots2, slots2_bytes, g, xa, sg, sxa, total;
  RankPlan g_plan, xa_plan, db_plan, da_plan;
};
BwdLayout bwd_layout(const LinearShape& s) {
  BwdLayout l{};
  l.g_plan = rank_tiling(s.m, s.rows, s.lora_steps);
  l.xa_plan = rank_tiling(s.m, s.cols, s.lora_steps);
  l.db_plan = rank_tiling(s.rows, s.m, s.lora_steps);
  l.da_plan = rank_tiling(s.cols, s.m, s.lora_steps);
  const int k1 = l.g_plan.ksteps > l.xa_plan.ksteps ? l.g_plan.ksteps : l.xa_plan.ksteps;
  const size_t alone = sized_slots(l.g_plan.tiles(), l.g_plan.ksteps);
  const size_t both = sized_slots(l.g_plan.tiles() + l.xa_plan.tiles(), k1);
  l.slots1_bytes = alone > both ? alone : both;
  l.slots2_bytes = s.decode ? 0 : sized_slots(l.db_plan.tiles() + l.da_plan.tiles(), l.db_plan.ksteps);
  size_t o = 0;
  l.cnt1 = o;   o = round_up(o + size_t(l.g_plan.tiles() + l.xa_plan.tiles()) * 4, 256);
  l.cnt2 = o;   o = round_up(o + size_t(l.db_plan.tiles() + l.da_plan.tiles()) * 4, 256);
  l.dx_acc = o; if (s.decode) o = round_up(o + size_t(s.m) * s.cols * 4, 256);
  l.clear_end = o;
  l.slots1 = o; o = round_up(o + l.slots1_bytes, 256);
  l.slots2 = o; o = round_up(o + l.slots2_bytes, 256);
  l.g = o;      if (s.decode) o = round_up(o + size_t(s.m) * s.rpad * 4, 256);
  l.xa = o;     if (s.decode) o = round_up(o + size_t(s.m) * s.rpad * 4, 256);
  l.sg = o;     o = round_up(o + size_t(s.m) * s.rpad * 2, 256);
  l.sxa = o;    o = round_up(o + size_t(s.m) * s.rpad * 2, 256);
  l.total = o;
  return l;
}

int choose_splits(int tiles, int ksteps, int num_sms) {
  int sp = (4 * num_sms + tiles - 1) / tiles;
  if (sp > ksteps) sp = ksteps;
  if (sp < 1) sp = 1;
  return sp;
}

// One rank-r problem of a k_rank launch.
RankProblem rank_problem(const RankPlan& pl, int64_t mdim, int64_t ndim, bool a_mn, bool b_mn, int unit_begin,
                         float* slots, uint32_t* counters) {
  RankProblem p{};
  p.mdim = mdim;
  p.ndim = ndim;
  p.ksteps = pl.ksteps;
  p.m_tiles = pl.m_tiles;
  p.n_tiles = pl.n_tiles;
  p.splits = pl.splits;
  p.unit_begin = unit_begin;
  p.a_mn = a_mn ? 1 : 0;
  p.b_mn = b_mn ? 1 : 0;
  p.slots = slots;
  p.counters = counters;
  return p;
}

// Decode-shaped forward (M <= 16): X A^T slices and the zeroed tile counters
// (k_xa_zero), then one pass over the packed weight that also writes Y
// (k_gemv, the programmatic dependent of k_xa_zero).  With adapter_idx each
// token uses its own adapter of the stacks A [n_adapters][r, cols] and
// B [n_adapters][rows, r].
qlora_status run_decode_fwd(const qlora_nf4_tensor* W, const uint16_t* X, const LinearShape& sh,
                            const uint16_t* A, const uint16_t* B, const int32_t* adapter_idx, int n_adapters,
                            float s, uint16_t* Y, float* XA_out, uint8_t* ws, const FwdLayout& L,
                            const DeviceInfo& d, cudaStream_t cs) {
  uint32_t* cnt = reinterpret_cast<uint32_t*>(ws + L.cnt);
  const int m_tiles = static_cast<int>((sh.rows + gemv_tile_rows() - 1) / gemv_tile_rows());
  float* xa_slices = reinterpret_cast<float*>(ws + L.xa_slices);
  const int xa_splits = xa_splits_for(sh.r, sh.cols);
  if (counted(launch_xa_zero(X, A, sh.m, sh.cols, sh.r, xa_slices, sh.rpad, xa_splits,
                             reinterpret_cast<float*>(cnt), static_cast<int64_t>(m_tiles) * 8, adapter_idx,
                             n_adapters, static_cast<int64_t>(sh.r) * sh.cols, d.err, cs)) != cudaSuccess)
    return QLORA_ERR_CUDA;
  CUtensorMap c_map, x_act;
  if (!make_map_u8(&c_map, W->codes, sh.cols / 2, sh.rows, sh.cols / 2, 128, gemv_tile_rows(),
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&x_act, X, sh.cols, sh.m, sh.cols * 2, static_cast<uint32_t>(sh.m)))
    return QLORA_ERR_CUDA;
  GemvArgs ga{};
  ga.qabs = W->absmax_q; ga.c2 = W->absmax_c2; ga.mean = W->absmax_mean;
  ga.absf = plain_absmax(W);
  ga.nw = sh.rows; ga.kw = sh.cols; ga.m = sh.m;
  ga.slots = reinterpret_cast<float*>(ws + L.slots);
  ga.cnt = cnt;
  ga.xa_part = xa_slices; ga.ld_xa = sh.rpad; ga.r = sh.r; ga.lora_steps = sh.lora_steps;
  ga.xa_splits = xa_splits;
  ga.s = s; ga.lora_b = B; ga.y = Y; ga.xa_out = XA_out;
  ga.adapter_idx = adapter_idx; ga.n_adapters = n_adapters; ga.b_stride = sh.rows * sh.r;
  ga.m_tiles = m_tiles;
  ga.steps = static_cast<int>((sh.cols / 64 + 3) / 4);
  const CodebookParam cbp = codebook_param(W->quant_type);
  for (int i = 0; i < 16; ++i) ga.level[i] = cbp.level[i];
  ga.err = d.err;
  if (counted(launch_gemv(ga, c_map, x_act, d.num_sms, cs)) != cudaSuccess) return QLORA_ERR_CUDA;
  return QLORA_OK;
}

}  // namespace

cudaError_t counted(cudaError_t e, int n) {
  if (e == cudaSuccess) g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed);
  return e;
}

qlora_status check_tensor(const qlora_nf4_tensor* t) {
  if (!t) return QLORA_ERR_NULL;
  if (t->rows < 0 || t->cols < 0 || t->rows > kMaxDim || t->cols > kMaxDim) return QLORA_ERR_SHAPE;
  if (t->blocksize != kBlock || (t->blocksize2 != kBlock2 && t->blocksize2 != 0)) return QLORA_ERR_UNSUPPORTED;
  if (t->quant_type < 0 || t->quant_type >= kNumTypes || t->reserved != 0) return QLORA_ERR_UNSUPPORTED;
  if (t->rows * t->cols == 0) return QLORA_OK;
  if (t->blocksize2 != 0) {          // double quantization: E4M3 codes, c2, mean
    if (!t->codes || !t->absmax_q || !t->absmax_c2 || !t->absmax_mean) return QLORA_ERR_NULL;
    if (!aligned16(t->codes) || !aligned16(t->absmax_q) || !aligned16(t->absmax_c2) ||
        !aligned16(t->absmax_mean))
      return QLORA_ERR_ALIGN;
  } else {                           // fp32 block constants
    if (!t->codes || !t->absmax) return QLORA_ERR_NULL;
    if (!aligned16(t->codes) || !aligned16(t->absmax)) return QLORA_ERR_ALIGN;
  }
  return QLORA_OK;
}

size_t quantize_workspace_bytes(int64_t numel, bool double_quant) {
  const int64_t nblocks = (numel + kBlock - 1) / kBlock;
  const size_t partials = kMaxEncodeGrid * sizeof(double);
  return double_quant ? round_up(static_cast<size_t>(nblocks) * 4, 256) + partials : partials;
}

EncodeTables encode_tables(const Nf4Tables& tabs) {
  EncodeTables et;
  for (int i = 0; i < kBuckets; ++i) {
    et.bucket_thr[i] = i < kNumBuckets ? tabs.bucket_thr[i] : INFINITY;
    et.bucket_base[i] = i < kNumBuckets ? tabs.bucket_base[i] : 15;
    et.bucket_fast[i] = i < kNumBuckets ? tabs.bucket_fast[i] : (0x7F7FFFE0u | 16u);
  }
  et.fast = tabs.fast_ok ? 1 : 0;
  return et;
}

qlora_status device_error_flag(uint32_t** flag) {
  DeviceInfo d;
  const qlora_status st = device_info(&d);
  if (st == QLORA_OK) *flag = d.err;
  return st;
}

}  // namespace qlora

using namespace qlora;

extern "C" {

const char* qlora_status_string(qlora_status s) {
  switch (s) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_NULL: return "null pointer";
    case QLORA_ERR_SHAPE: return "unsupported shape";
    case QLORA_ERR_ALIGN: return "pointer not 16-byte aligned";
    case QLORA_ERR_UNSUPPORTED: return "unsupported configuration or device";
    case QLORA_ERR_CUDA: return "CUDA error";
    case QLORA_ERR_WORKSPACE: return "work buffer too small";
  }
  return "unknown status";
}

void qlora_get_codebook(float out[16]) {
  if (!out) return;
  const Nf4Tables& t = nf4_tables();
  for (int i = 0; i < 16; ++i) out[i] = t.level[i];
}

qlora_status qlora_get_levels(int32_t quant_type, float out[16]) {
  if (!out) return QLORA_ERR_NULL;
  if (quant_type < 0 || quant_type >= kNumTypes) return QLORA_ERR_UNSUPPORTED;
  const Nf4Tables& t = level_tables(quant_type);
  for (int i = 0; i < 16; ++i) out[i] = t.level[i];
  return QLORA_OK;
}

qlora_status qlora_nf4_sizes(int64_t rows, int64_t cols, int32_t blocksize, int32_t blocksize2,
                             size_t* codes_bytes, size_t* absmax_q_bytes, size_t* absmax_c2_bytes,
                             size_t* workspace_bytes) {
  if (rows < 0 || cols < 0 || rows > kMaxDim || cols > kMaxDim) return QLORA_ERR_SHAPE;
  if (blocksize != kBlock || (blocksize2 != kBlock2 && blocksize2 != 0)) return QLORA_ERR_UNSUPPORTED;
  const bool dq = blocksize2 != 0;
  const int64_t numel = rows * cols;
  const int64_t nblocks = (numel + kBlock - 1) / kBlock;
  const int64_t ngroups = (nblocks + kBlock2 - 1) / kBlock2;
  if (codes_bytes) *codes_bytes = static_cast<size_t>((numel + 1) / 2);
  if (absmax_q_bytes) *absmax_q_bytes = static_cast<size_t>(nblocks) * (dq ? 1 : 4);
  if (absmax_c2_bytes) *absmax_c2_bytes = dq ? static_cast<size_t>(ngroups) * 4 : 0;
  if (workspace_bytes) *workspace_bytes = quantize_workspace_bytes(numel, dq);
  return QLORA_OK;
}

qlora_status qlora_quantize_nf4_dq(const uint16_t* W, const qlora_nf4_tensor* out, void* workspace,
                                   size_t workspace_bytes, qlora_stream_t stream) {
  qlora_status st = check_tensor(out);
  if (st != QLORA_OK) return st;
  const int64_t numel = out->rows * out->cols;
  if (numel == 0) return QLORA_OK;
  if (!W || !workspace) return QLORA_ERR_NULL;
  if (!aligned16(W) || !aligned16(workspace)) return QLORA_ERR_ALIGN;
  const bool dq = out->blocksize2 != 0;
  if (workspace_bytes < quantize_workspace_bytes(numel, dq)) return QLORA_ERR_WORKSPACE;
  const Nf4Tables& tabs = level_tables(out->quant_type);
  if (!tabs.ok) return QLORA_ERR_UNSUPPORTED;
  DeviceInfo d;
  if ((st = device_info(&d)) != QLORA_OK) return st;

  const EncodeTables et = encode_tables(tabs);
  const int64_t nblocks = (numel + kBlock - 1) / kBlock;
  // with double quantization the block absmax values are scratch for
  // k_double_quant; without it they are the stored constants themselves
  float* c1buf = dq ? static_cast<float*>(workspace) : out->absmax;
  double* partials = reinterpret_cast<double*>(
      static_cast<uint8_t*>(workspace) + (dq ? round_up(static_cast<size_t>(nblocks) * 4, 256) : 0));
  const int64_t nvec = nblocks * 8;
  int grid = static_cast<int>((nvec + 255) / 256);
  const int wave = d.num_sms * encode_ctas_per_sm();           // one wave of resident CTAs
  const int cap = wave < kMaxEncodeGrid ? wave : kMaxEncodeGrid;
  if (grid > cap) grid = cap;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = counted(launch_encode(W, numel, et, out->codes, c1buf, partials, grid, s));
  if (e != cudaSuccess) return QLORA_ERR_CUDA;
  if (!dq) return QLORA_OK;
  const int64_t ngroups = (nblocks + kBlock2 - 1) / kBlock2;
  int grid2 = static_cast<int>((ngroups + 7) / 8);
  if (grid2 > d.num_sms * 4) grid2 = d.num_sms * 4;
  if (grid2 < 1) grid2 = 1;
  e = counted(launch_double_quant(c1buf, nblocks, partials, grid, out->absmax_q, out->absmax_c2,
                                  out->absmax_mean, grid2, s));
  return cuda_status(e);
}

qlora_status qlora_dequantize(const qlora_nf4_tensor* W, uint16_t* W_out, qlora_stream_t stream) {
  qlora_status st = check_tensor(W);
  if (st != QLORA_OK) return st;
  const int64_t numel = W->rows * W->cols;
  if (numel == 0) return QLORA_OK;
  if (!W_out) return QLORA_ERR_NULL;
  if (!aligned16(W_out)) return QLORA_ERR_ALIGN;
  DeviceInfo d;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  const int64_t nchunks = (numel + 31) / 32;
  int grid = static_cast<int>((nchunks + 255) / 256);
  const int wave = d.num_sms * dequant_ctas_per_sm();          // one wave of resident CTAs
  if (grid > wave) grid = wave;
  return cuda_status(counted(launch_dequant(W->codes, W->absmax_q, W->absmax_c2, W->absmax_mean,
                                            plain_absmax(W), numel, codebook_param(W->quant_type), W_out, grid,
                                            reinterpret_cast<cudaStream_t>(stream))));
}

qlora_status qlora_linear_workspace_size(int64_t rows, int64_t cols, int64_t M, int32_t r,
                                         size_t* fwd_bytes, size_t* bwd_bytes) {
  if (rows < 8 || cols < 64 || rows > kMaxDim || cols > kMaxDim || cols % 64 || rows % 8)
    return QLORA_ERR_SHAPE;
  if (M < 1 || M > kMaxDim || r < 8 || r > 256 || r % 8) return QLORA_ERR_SHAPE;
  LinearShape sh;
  sh.rows = rows;
  sh.cols = cols;
  sh.m = M;
  sh.r = r;
  sh.lora_steps = (r + 63) / 64;
  sh.rpad = 64 * sh.lora_steps;
  sh.decode = M <= 16;
  if (fwd_bytes) *fwd_bytes = fwd_layout(sh).total;
  if (bwd_bytes) *bwd_bytes = bwd_layout(sh).total;
  return QLORA_OK;
}

qlora_status qlora_linear_fwd(const qlora_nf4_tensor* W, const uint16_t* X, int64_t M,
                              const uint16_t* A, const uint16_t* B, int32_t r, float s, uint16_t* Y,
                              float* XA_out, void* workspace, size_t workspace_bytes,
                              qlora_stream_t stream) {
  LinearShape sh;
  qlora_status st = check_linear(W, M, r, &sh);
  if (st != QLORA_OK) return st;
  if (!X || !A || !B || !Y || !workspace) return QLORA_ERR_NULL;
  if (!aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(Y) || !aligned16(workspace) ||
      (XA_out && !aligned16(XA_out)))
    return QLORA_ERR_ALIGN;
  if (!std::isfinite(s)) return QLORA_ERR_SHAPE;
  const FwdLayout L = fwd_layout(sh);
  if (workspace_bytes < L.total) return QLORA_ERR_WORKSPACE;
  DeviceInfo d;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  if (sh.decode)
    return run_decode_fwd(W, X, sh, A, B, nullptr, 1, s, Y, XA_out, ws, L, d, cs);

  // 1) X A^T (fp32 to XA_out when asked) and bf16(s X A^T), zero-padded to a
  //    multiple of 64 columns, as the LoRA k-step operand of the fused GEMM
  uint16_t* sxa = reinterpret_cast<uint16_t*>(ws + L.sxa);
  RankPlan xp = rank_tiling(sh.m, sh.cols, sh.lora_steps);
  xp.splits = launch_splits(xp.tiles(), xp.ksteps, d.num_sms, L.rank_slot_bytes);
  if (!slots_fit(xp.tiles(), xp.splits, L.rank_slot_bytes)) return QLORA_ERR_WORKSPACE;
  if (xp.splits > 1 && cudaMemsetAsync(ws, 0, L.clear_end, cs) != cudaSuccess) return QLORA_ERR_CUDA;
  CUtensorMap x_k, a_k;
  if (!make_map(&x_k, X, sh.cols, sh.m, sh.cols * 2, 128) ||
      !make_map(&a_k, A, sh.cols, sh.r, sh.cols * 2, 64))
    return QLORA_ERR_CUDA;
  RankArgs ra{};
  ra.p[0] = rank_problem(xp, sh.m, sh.r, false, false, 0, reinterpret_cast<float*>(ws + L.rank_slots),
                         reinterpret_cast<uint32_t*>(ws + L.rank_cnt));
  ra.p[0].out_f32 = XA_out; ra.p[0].ld_f32 = sh.r;
  ra.p[0].out_bf16 = sxa; ra.p[0].ld_bf16 = sh.rpad; ra.p[0].bf16_cols = sh.rpad; ra.p[0].bf16_scale = s;
  ra.nprob = 1;
  ra.total_units = xp.tiles() * xp.splits;
  ra.err = d.err;
  if (counted(launch_rank(ra, x_k, a_k, x_k, a_k, d.num_sms, cs)) != cudaSuccess) return QLORA_ERR_CUDA;

  // 2) Y = X deq(W)^T + (s XA) B^T  (fused dequant GEMM)
  const int bn = 256;
  CUtensorMap x_act, sxa_map;
  if (!make_map(&x_act, X, sh.cols, sh.m, sh.cols * 2, bn) ||
      !make_map(&sxa_map, sxa, sh.rpad, sh.m, sh.rpad * 2, bn))
    return QLORA_ERR_CUDA;
  FusedArgs fa{};
  fa.codes = W->codes; fa.qabs = W->absmax_q; fa.c2 = W->absmax_c2; fa.mean = W->absmax_mean;
  fa.absf = plain_absmax(W);
  fa.nw = sh.rows; fa.kw = sh.cols; fa.m = sh.m;
  fa.lora_w = B; fa.r = sh.r; fa.lora_steps = sh.lora_steps;
  fa.ldo = sh.rows; fa.mdim = sh.rows;
  fa.ksteps = static_cast<int>(sh.cols / 64);
  fa.m_tiles = static_cast<int>((sh.rows + 127) / 128);
  fa.t_tiles = static_cast<int>((sh.m + bn - 1) / bn);
  fa.splits = 1;
  fa.m_group = m_group_for(fa.m_tiles, sh.cols);
  fa.out = Y; fa.out_acc = nullptr;
  fa.cb = codebook_param(W->quant_type);
  fa.err = d.err;
  if (fused_timed(FusedDir::kFwd, bn, fa, x_act, sxa_map, d.num_sms, cs) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return QLORA_OK;
}

qlora_status qlora_linear_fwd_multi(const qlora_nf4_tensor* W, const uint16_t* X, int64_t M,
                                    const uint16_t* A_stack, const uint16_t* B_stack, int32_t n_adapters,
                                    const int32_t* adapter_idx, int32_t r, float s, uint16_t* Y,
                                    float* XA_out, void* workspace, size_t workspace_bytes,
                                    qlora_stream_t stream) {
  LinearShape sh;
  qlora_status st = check_linear(W, M, r, &sh);
  if (st != QLORA_OK) return st;
  if (!sh.decode || n_adapters < 1) return QLORA_ERR_SHAPE;
  if (!X || !A_stack || !B_stack || !adapter_idx || !Y || !workspace) return QLORA_ERR_NULL;
  if (!aligned16(X) || !aligned16(A_stack) || !aligned16(B_stack) || !aligned16(Y) || !aligned16(workspace) ||
      (XA_out && !aligned16(XA_out)) || (reinterpret_cast<uintptr_t>(adapter_idx) & 3u) != 0)
    return QLORA_ERR_ALIGN;
  if (!std::isfinite(s)) return QLORA_ERR_SHAPE;
  const FwdLayout L = fwd_layout(sh);
  if (workspace_bytes < L.total) return QLORA_ERR_WORKSPACE;
  DeviceInfo d;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  return run_decode_fwd(W, X, sh, A_stack, B_stack, adapter_idx, n_adapters, s, Y, XA_out,
                        static_cast<uint8_t*>(workspace), L, d, reinterpret_cast<cudaStream_t>(stream));
}

qlora_status qlora_linear_bwd(const qlora_nf4_tensor* W, const uint16_t* X, const uint16_t* dY,
                              int64_t M, const uint16_t* A, const uint16_t* B, int32_t r, float s,
                              const float* XA, uint16_t* dX, float* dA, float* dB,
                              void* workspace, size_t workspace_bytes, qlora_stream_t stream) {
  LinearShape sh;
  qlora_status st = check_linear(W, M, r, &sh);
  if (st != QLORA_OK) return st;
  if (!X || !dY || !A || !B || !dA || !dB || !workspace) return QLORA_ERR_NULL;
  if (!aligned16(X) || !aligned16(dY) || !aligned16(A) || !aligned16(B) || !aligned16(dA) ||
      !aligned16(dB) || !aligned16(workspace) || (XA && !aligned16(XA)) || (dX && !aligned16(dX)))
    return QLORA_ERR_ALIGN;
  if (!std::isfinite(s)) return QLORA_ERR_SHAPE;
  BwdLayout L = bwd_layout(sh);
  if (workspace_bytes < L.total) return QLORA_ERR_WORKSPACE;
  DeviceInfo d;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* dx_acc = reinterpret_cast<float*>(ws + L.dx_acc);
  float* g32 = sh.decode ? reinterpret_cast<float*>(ws + L.g) : nullptr;     // fp32 G and X A^T: few-token grads
  float* xa32 = sh.decode ? reinterpret_cast<float*>(ws + L.xa) : nullptr;
  uint16_t* sg = reinterpret_cast<uint16_t*>(ws + L.sg);
  uint16_t* sxa = reinterpret_cast<uint16_t*>(ws + L.sxa);
  const bool recompute = XA == nullptr;

  if (L.clear_end && cudaMemsetAsync(ws, 0, L.clear_end, cs) != cudaSuccess) return QLORA_ERR_CUDA;

  // 1) G = dY B -> bf16(s G) (+ fp32 G for few tokens), and X A^T -> bf16(s X A^T)
  //    (recomputed when not supplied, else converted from the caller's fp32)
  CUtensorMap dy_k, b_mn, x_k, a_k;
  if (!make_map(&dy_k, dY, sh.rows, sh.m, sh.rows * 2, 128) ||
      !make_map(&b_mn, B, sh.r, sh.rows, sh.r * 2, 64) ||
      !make_map(&x_k, X, sh.cols, sh.m, sh.cols * 2, 128) ||
      !make_map(&a_k, A, sh.cols, sh.r, sh.cols * 2, 64))
    return QLORA_ERR_CUDA;
  {
    // splits for this device and this form of launch 1, within the slot space
    if (recompute) {
      const int k1 = L.g_plan.ksteps > L.xa_plan.ksteps ? L.g_plan.ksteps : L.xa_plan.ksteps;
      L.g_plan.splits = L.xa_plan.splits =
          launch_splits(L.g_plan.tiles() + L.xa_plan.tiles(), k1, d.num_sms, L.slots1_bytes);
    } else {
      L.g_plan.splits = launch_splits(L.g_plan.tiles(), L.g_plan.ksteps, d.num_sms, L.slots1_bytes);
    }
    if (!slots_fit(L.g_plan.tiles() + (recompute ? L.xa_plan.tiles() : 0), L.g_plan.splits, L.slots1_bytes))
      return QLORA_ERR_WORKSPACE;
    RankArgs ra{};
    uint32_t* cnt = reinterpret_cast<uint32_t*>(ws + L.cnt1);
    float* slots = reinterpret_cast<float*>(ws + L.slots1);
    ra.p[0] = rank_problem(L.g_plan, sh.m, sh.r, false, true, 0, slots, cnt);
    ra.p[0].out_f32 = g32; ra.p[0].ld_f32 = sh.rpad;
    ra.p[0].out_bf16 = sg; ra.p[0].ld_bf16 = sh.rpad; ra.p[0].bf16_cols = sh.rpad; ra.p[0].bf16_scale = s;
    ra.nprob = 1;
    ra.total_units = L.g_plan.tiles() * L.g_plan.splits;
    if (recompute) {
      ra.p[1] = rank_problem(L.xa_plan, sh.m, sh.r, false, false, ra.total_units,
                             slots + rank_slot_bytes(L.g_plan.tiles(), L.g_plan.splits) / 4,
                             cnt + L.g_plan.tiles());
      ra.p[1].out_f32 = xa32; ra.p[1].ld_f32 = sh.rpad;
      ra.p[1].out_bf16 = sh.decode ? nullptr : sxa;
      ra.p[1].ld_bf16 = sh.rpad; ra.p[1].bf16_cols = sh.rpad; ra.p[1].bf16_scale = s;
      ra.nprob = 2;
      ra.total_units += L.xa_plan.tiles() * L.xa_plan.splits;
    } else if (!sh.decode) {
      ra.cvt_in = XA; ra.cvt_rows = sh.m; ra.cvt_cols = sh.r; ra.cvt_ld_in = sh.r;
      ra.cvt_out = sxa; ra.cvt_ld_out = sh.rpad; ra.cvt_cols_out = sh.rpad; ra.cvt_scale = s;
    }
    ra.err = d.err;
    if (counted(launch_rank(ra, dy_k, b_mn, x_k, a_k, d.num_sms, cs)) != cudaSuccess) return QLORA_ERR_CUDA;
  }

  // 2) dX = dY deq(W) + (s G) A   (fused dequant GEMM, deq(W)^T as the MN-major operand)
  if (dX) {
    const int bn = sh.decode ? 16 : 256;
    CUtensorMap dy_act, sg_map;
    if (!make_map(&dy_act, dY, sh.rows, sh.m, sh.rows * 2, bn) ||
        !make_map(&sg_map, sg, sh.rpad, sh.m, sh.rpad * 2, bn))
      return QLORA_ERR_CUDA;
    FusedArgs fa{};
    fa.codes = W->codes; fa.qabs = W->absmax_q; fa.c2 = W->absmax_c2; fa.mean = W->absmax_mean;
    fa.absf = plain_absmax(W);
    fa.nw = sh.rows; fa.kw = sh.cols; fa.m = sh.m;
    fa.lora_w = A; fa.r = sh.r; fa.lora_steps = sh.lora_steps;
    fa.ldo = sh.cols; fa.mdim = sh.cols;
    fa.ksteps = static_cast<int>((sh.rows + 63) / 64);
    fa.m_tiles = static_cast<int>((sh.cols + 127) / 128);
    fa.t_tiles = static_cast<int>((sh.m + bn - 1) / bn);
    fa.splits = sh.decode ? choose_splits(fa.m_tiles, fa.ksteps, d.num_sms) : 1;
    fa.m_group = m_group_for(fa.m_tiles, sh.rows);
    fa.out = dX; fa.out_acc = dx_acc;
    fa.cb = codebook_param(W->quant_type);
    fa.err = d.err;
    if (fused_timed(FusedDir::kBwd, bn, fa, dy_act, sg_map, d.num_sms, cs) != cudaSuccess)
      return QLORA_ERR_CUDA;
    if (fa.splits > 1 &&
        counted(launch_convert_bf16(dx_acc, sh.m, sh.cols, sh.cols, sh.cols, 1.0f, dX, sh.cols, d.num_sms, cs)) !=
            cudaSuccess)
      return QLORA_ERR_CUDA;
  }

  // 3) LoRA gradients.  Few tokens: fp32 on CUDA cores from the fp32 G and X A^T.
  if (sh.decode) {
    const float* xa = recompute ? xa32 : XA;
    const int64_t ld_xa = recompute ? sh.rpad : sh.r;
    if (counted(launch_small_grads(g32, sh.rpad, xa, ld_xa, X, dY, sh.m, sh.rows, sh.cols, sh.r, s,
                                   dA, dB, d.num_sms, cs)) != cudaSuccess)
      return QLORA_ERR_CUDA;
    return QLORA_OK;
  }
  //    Many tokens, one launch of two contractions over the tokens (bf16 operands):
  //    dB = dY^T (s X A^T) [rows, r] and dA = (X^T (s G))^T [r, cols], stored transposed.
  CUtensorMap dy_mn, sxa_mn, x_mn, sg_mn;
  if (!make_map(&dy_mn, dY, sh.rows, sh.m, sh.rows * 2, 64) ||
      !make_map(&sxa_mn, sxa, sh.rpad, sh.m, sh.rpad * 2, 64) ||
      !make_map(&x_mn, X, sh.cols, sh.m, sh.cols * 2, 64) ||
      !make_map(&sg_mn, sg, sh.rpad, sh.m, sh.rpad * 2, 64))
    return QLORA_ERR_CUDA;
  L.db_plan.splits = L.da_plan.splits =
      launch_splits(L.db_plan.tiles() + L.da_plan.tiles(), L.db_plan.ksteps, d.num_sms, L.slots2_bytes);
  if (!slots_fit(L.db_plan.tiles() + L.da_plan.tiles(), L.db_plan.splits, L.slots2_bytes))
    return QLORA_ERR_WORKSPACE;
  RankArgs rb{};
  uint32_t* cnt2 = reinterpret_cast<uint32_t*>(ws + L.cnt2);
  float* slots2 = reinterpret_cast<float*>(ws + L.slots2);
  rb.p[0] = rank_problem(L.db_plan, sh.rows, sh.r, true, true, 0, slots2, cnt2);
  rb.p[0].out_f32 = dB; rb.p[0].ld_f32 = sh.r;
  const int u0 = L.db_plan.tiles() * L.db_plan.splits;
  rb.p[1] = rank_problem(L.da_plan, sh.cols, sh.r, true, true, u0,
                         slots2 + rank_slot_bytes(L.db_plan.tiles(), L.db_plan.splits) / 4,
                         cnt2 + L.db_plan.tiles());
  rb.p[1].out_f32 = dA; rb.p[1].ld_f32 = sh.cols; rb.p[1].transpose = 1;
  rb.nprob = 2;
  rb.total_units = u0 + L.da_plan.tiles() * L.da_plan.splits;
  rb.err = d.err;
  if (counted(launch_rank(rb, dy_mn, sxa_mn, x_mn, sg_mn, d.num_sms, cs)) != cudaSuccess) return QLORA_ERR_CUDA;
  return QLORA_OK;
}

qlora_status qlora_read_device_errors(uint32_t* flags, int clear) {
  if (!flags) return QLORA_ERR_NULL;
  DeviceInfo d;
  qlora_status st = device_info(&d);
  if (st != QLORA_OK) return st;
  if (cudaMemcpy(flags, d.err, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return QLORA_ERR_CUDA;
  if (clear && cudaMemset(d.err, 0, 4) != cudaSuccess) return QLORA_ERR_CUDA;
  return QLORA_OK;
}

uint64_t qlora_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

qlora_status qlora_time_next_gemm(void* start_event, void* stop_event) {
  if ((start_event == nullptr) != (stop_event == nullptr)) return QLORA_ERR_NULL;
  t_gemm_start = static_cast<cudaEvent_t>(start_event);
  t_gemm_stop = static_cast<cudaEvent_t>(stop_event);
  return QLORA_OK;
}

}  // extern "C"
