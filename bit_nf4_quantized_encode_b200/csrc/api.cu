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

cudaError_t fused_timed(FusedDir dir, int bn, const FusedArgs& fa, const CUtensorMap& act,
                        const CUtensorMap& lora, int num_sms, cudaStream_t cs) {
  cudaEvent_t e0 = t_gemm_start, e1 = t_gemm_stop;
  t_gemm_start = t_gemm_stop = nullptr;
  if (e0 && cudaEventRecord(e0, cs) != cudaSuccess) return cudaErrorUnknown;
  cudaError_t e = counted(launch_fused(dir, bn, fa, act, lora, num_sms, cs));
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

CodebookParam codebook_param() {
  CodebookParam cb;
  const Nf4Tables& t = nf4_tables();
  for (int i = 0; i < 16; ++i) cb.level[i] = t.level[i];
  return cb;
}

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
struct FwdLayout {
  size_t xa_acc, cnt, slots, fp32_end, sxa, xa_slices, total;
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
    l.fp32_end = 0;
    l.total = o;
    return l;
  }
  l.xa_acc = o; o = round_up(o + size_t(s.m) * s.rpad * 4, 256);
  l.fp32_end = o;
  l.sxa = o;    o = round_up(o + size_t(s.m) * s.rpad * 2, 256);
  l.total = o;
  return l;
}

struct BwdLayout {
  size_t g_acc, xa_acc, dx_acc, da_acc, db_acc, fp32_end, sg, xa, total;
};
BwdLayout bwd_layout(const LinearShape& s) {
  BwdLayout l{};
  size_t o = 0;
  l.g_acc = o;  o = round_up(o + size_t(s.m) * s.rpad * 4, 256);
  l.xa_acc = o; o = round_up(o + size_t(s.m) * s.rpad * 4, 256);
  l.dx_acc = o; if (s.decode) o = round_up(o + size_t(s.m) * s.cols * 4, 256);
  l.da_acc = o; o = round_up(o + size_t(s.cols) * s.rpad * 4, 256);
  l.db_acc = o; o = round_up(o + size_t(s.rows) * s.rpad * 4, 256);
  l.fp32_end = o;
  l.sg = o;     o = round_up(o + size_t(s.m) * s.rpad * 2, 256);
  l.xa = o;     o = round_up(o + size_t(s.m) * s.rpad * 2, 256);
  l.total = o;
  return l;
}

int choose_splits(int tiles, int ksteps, int num_sms) {
  int s = (4 * num_sms + tiles - 1) / tiles;
  if (s > ksteps) s = ksteps;
  if (s < 1) s = 1;
  return s;
}

// D[mdim, ndim] (+)= A B^T over kdim; A and B as tensor maps; fp32 acc.
qlora_status run_skinny(bool a_mn, bool b_mn, const CUtensorMap& am, const CUtensorMap& bm,
                        int64_t mdim, int64_t ndim, int64_t kdim, float* acc, int64_t ld_acc,
                        const DeviceInfo& d, cudaStream_t stream) {
  SkinnyArgs sa{};
  sa.mdim = mdim;
  sa.ndim = ndim;
  sa.ksteps = static_cast<int>((kdim + 63) / 64);
  sa.m_tiles = static_cast<int>((mdim + 127) / 128);
  sa.n_tiles = static_cast<int>((ndim + 63) / 64);
  sa.splits = choose_splits(sa.m_tiles * sa.n_tiles, sa.ksteps, d.num_sms);
  sa.acc = acc;
  sa.ld_acc = ld_acc;
  sa.err = d.err;
  return cuda_status(counted(launch_skinny(a_mn, b_mn, sa, am, bm, d.num_sms, stream)));
}

}  // namespace

cudaError_t counted(cudaError_t e, int n) {
  if (e == cudaSuccess) g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed);
  return e;
}

qlora_status check_tensor(const qlora_nf4_tensor* t) {
  if (!t) return QLORA_ERR_NULL;
  if (t->rows < 0 || t->cols < 0 || t->rows > kMaxDim || t->cols > kMaxDim) return QLORA_ERR_SHAPE;
  if (t->blocksize != kBlock || t->blocksize2 != kBlock2) return QLORA_ERR_UNSUPPORTED;
  if (t->rows * t->cols == 0) return QLORA_OK;
  if (!t->codes || !t->absmax_q || !t->absmax_c2 || !t->absmax_mean) return QLORA_ERR_NULL;
  if (!aligned16(t->codes) || !aligned16(t->absmax_q) || !aligned16(t->absmax_c2) ||
      !aligned16(t->absmax_mean))
    return QLORA_ERR_ALIGN;
  return QLORA_OK;
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

qlora_status qlora_nf4_sizes(int64_t rows, int64_t cols, int32_t blocksize, int32_t blocksize2,
                             size_t* codes_bytes, size_t* absmax_q_bytes, size_t* absmax_c2_bytes,
                             size_t* workspace_bytes) {
  if (rows < 0 || cols < 0 || rows > kMaxDim || cols > kMaxDim) return QLORA_ERR_SHAPE;
  if (blocksize != kBlock || blocksize2 != kBlock2) return QLORA_ERR_UNSUPPORTED;
  const int64_t numel = rows * cols;
  const int64_t nblocks = (numel + kBlock - 1) / kBlock;
  const int64_t ngroups = (nblocks + kBlock2 - 1) / kBlock2;
  if (codes_bytes) *codes_bytes = static_cast<size_t>((numel + 1) / 2);
  if (absmax_q_bytes) *absmax_q_bytes = static_cast<size_t>(nblocks);
  if (absmax_c2_bytes) *absmax_c2_bytes = static_cast<size_t>(ngroups) * 4;
  if (workspace_bytes)
    *workspace_bytes = round_up(static_cast<size_t>(nblocks) * 4, 256) + kMaxEncodeGrid * sizeof(double);
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
  size_t need = 0;
  qlora_nf4_sizes(out->rows, out->cols, kBlock, kBlock2, nullptr, nullptr, nullptr, &need);
  if (workspace_bytes < need) return QLORA_ERR_WORKSPACE;
  const Nf4Tables& tabs = nf4_tables();
  if (!tabs.ok) return QLORA_ERR_UNSUPPORTED;
  DeviceInfo d;
  if ((st = device_info(&d)) != QLORA_OK) return st;

  EncodeTables et;
  for (int i = 0; i < kBuckets; ++i) {
    et.bucket_thr[i] = i < kNumBuckets ? tabs.bucket_thr[i] : INFINITY;
    et.bucket_base[i] = i < kNumBuckets ? tabs.bucket_base[i] : 15;
    et.bucket_fast[i] = i < kNumBuckets ? tabs.bucket_fast[i] : (0x7F7FFFE0u | 16u);
  }
  et.fast = tabs.fast_ok ? 1 : 0;

  const int64_t nblocks = (numel + kBlock - 1) / kBlock;
  float* c1buf = static_cast<float*>(workspace);
  double* partials = reinterpret_cast<double*>(static_cast<uint8_t*>(workspace) +
                                               round_up(static_cast<size_t>(nblocks) * 4, 256));
  const int64_t nvec = nblocks * 8;
  int grid = static_cast<int>((nvec + 255) / 256);
  const int wave = d.num_sms * encode_ctas_per_sm();           // one wave of resident CTAs
  const int cap = wave < kMaxEncodeGrid ? wave : kMaxEncodeGrid;
  if (grid > cap) grid = cap;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = counted(launch_encode(W, numel, et, out->codes, c1buf, partials, grid, s));
  if (e != cudaSuccess) return QLORA_ERR_CUDA;
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
                                            numel, codebook_param(), W_out, grid,
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

  if (sh.decode) {
    // Decode shapes: X A^T slices and the zeroed tile counters (k_xa_zero),
    // then one pass over the packed weight that also writes Y (k_gemv, the
    // programmatic dependent of k_xa_zero).
    uint32_t* cnt = reinterpret_cast<uint32_t*>(ws + L.cnt);
    const int m_tiles = static_cast<int>((sh.rows + gemv_tile_rows() - 1) / gemv_tile_rows());
    float* xa_slices = reinterpret_cast<float*>(ws + L.xa_slices);
    const int xa_splits = xa_splits_for(sh.r, sh.cols);
    if (counted(launch_xa_zero(X, A, sh.m, sh.cols, sh.r, xa_slices, sh.rpad, xa_splits,
                               reinterpret_cast<float*>(cnt), static_cast<int64_t>(m_tiles) * 8, cs)) !=
        cudaSuccess)
      return QLORA_ERR_CUDA;
    CUtensorMap c_map, x_act;
    if (!make_map_u8(&c_map, W->codes, sh.cols / 2, sh.rows, sh.cols / 2, 128, gemv_tile_rows(),
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&x_act, X, sh.cols, sh.m, sh.cols * 2, static_cast<uint32_t>(sh.m)))
      return QLORA_ERR_CUDA;
    GemvArgs ga{};
    ga.qabs = W->absmax_q; ga.c2 = W->absmax_c2; ga.mean = W->absmax_mean;
    ga.nw = sh.rows; ga.kw = sh.cols; ga.m = sh.m;
    ga.slots = reinterpret_cast<float*>(ws + L.slots);
    ga.cnt = cnt;
    ga.xa_part = xa_slices; ga.ld_xa = sh.rpad; ga.r = sh.r; ga.lora_steps = sh.lora_steps;
    ga.xa_splits = xa_splits;
    ga.s = s; ga.lora_b = B; ga.y = Y; ga.xa_out = XA_out;
    ga.m_tiles = m_tiles;
    ga.steps = static_cast<int>((sh.cols / 64 + 3) / 4);
    const CodebookParam cbp = codebook_param();
    for (int i = 0; i < 16; ++i) ga.level[i] = cbp.level[i];
    ga.err = d.err;
    if (counted(launch_gemv(ga, c_map, x_act, d.num_sms, cs)) != cudaSuccess) return QLORA_ERR_CUDA;
    return QLORA_OK;
  }

  float* xa_acc = reinterpret_cast<float*>(ws + L.xa_acc);
  uint16_t* sxa = reinterpret_cast<uint16_t*>(ws + L.sxa);
  if (cudaMemsetAsync(ws, 0, L.fp32_end, cs) != cudaSuccess) return QLORA_ERR_CUDA;

  // 1) XA = X A^T  (skinny tcgen05 GEMM, split-K into fp32)
  CUtensorMap x_k, a_k;
  if (!make_map(&x_k, X, sh.cols, sh.m, sh.cols * 2, 128) ||
      !make_map(&a_k, A, sh.cols, sh.r, sh.cols * 2, 64))
    return QLORA_ERR_CUDA;
  if ((st = run_skinny(false, false, x_k, a_k, sh.m, sh.r, sh.cols, xa_acc, sh.rpad, d, cs)) != QLORA_OK)
    return st;
  // 2) bf16(s XA), zero-padded to a multiple of 64 columns, as the LoRA k-step operand;
  //    XA itself (fp32, unscaled) for the backward pass
  if (counted(launch_convert_bf16(xa_acc, sh.m, sh.rpad, sh.rpad, sh.rpad, s, sxa, sh.rpad, d.num_sms, cs)) !=
      cudaSuccess)
    return QLORA_ERR_CUDA;
  if (XA_out &&
      counted(launch_convert_f32(xa_acc, sh.m, sh.r, sh.rpad, 1.0f, false, XA_out, sh.r, d.num_sms, cs)) !=
          cudaSuccess)
    return QLORA_ERR_CUDA;

  // 3) Y = X deq(W)^T + (s XA) B^T  (fused dequant GEMM)
  const int bn = sh.decode ? 16 : 256;
  CUtensorMap x_act, sxa_map;
  if (!make_map(&x_act, X, sh.cols, sh.m, sh.cols * 2, bn) ||
      !make_map(&sxa_map, sxa, sh.rpad, sh.m, sh.rpad * 2, bn))
    return QLORA_ERR_CUDA;
  FusedArgs fa{};
  fa.codes = W->codes; fa.qabs = W->absmax_q; fa.c2 = W->absmax_c2; fa.mean = W->absmax_mean;
  fa.nw = sh.rows; fa.kw = sh.cols; fa.m = sh.m;
  fa.lora_w = B; fa.r = sh.r; fa.lora_steps = sh.lora_steps;
  fa.ldo = sh.rows; fa.mdim = sh.rows;
  fa.ksteps = static_cast<int>(sh.cols / 64);
  fa.m_tiles = static_cast<int>((sh.rows + 127) / 128);
  fa.t_tiles = static_cast<int>((sh.m + bn - 1) / bn);
  fa.splits = 1;
  fa.m_group = m_group_for(fa.m_tiles, sh.cols);
  fa.out = Y; fa.out_acc = nullptr;
  fa.cb = codebook_param();
  fa.err = d.err;
  if (fused_timed(FusedDir::kFwd, bn, fa, x_act, sxa_map, d.num_sms, cs) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return QLORA_OK;
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
  const BwdLayout L = bwd_layout(sh);
  if (workspace_bytes < L.total) return QLORA_ERR_WORKSPACE;
  DeviceInfo d;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* g_acc = reinterpret_cast<float*>(ws + L.g_acc);
  float* xa_acc = reinterpret_cast<float*>(ws + L.xa_acc);
  float* dx_acc = reinterpret_cast<float*>(ws + L.dx_acc);
  float* da_acc = reinterpret_cast<float*>(ws + L.da_acc);
  float* db_acc = reinterpret_cast<float*>(ws + L.db_acc);
  uint16_t* sg = reinterpret_cast<uint16_t*>(ws + L.sg);
  uint16_t* sxa = reinterpret_cast<uint16_t*>(ws + L.xa);

  if (cudaMemsetAsync(ws, 0, L.fp32_end, cs) != cudaSuccess) return QLORA_ERR_CUDA;

  // 1) G = dY B   (contraction over rows; B [rows, r] is the MN-major operand)
  CUtensorMap dy_k, b_mn;
  if (!make_map(&dy_k, dY, sh.rows, sh.m, sh.rows * 2, 128) ||
      !make_map(&b_mn, B, sh.r, sh.rows, sh.r * 2, 64))
    return QLORA_ERR_CUDA;
  if ((st = run_skinny(false, true, dy_k, b_mn, sh.m, sh.r, sh.rows, g_acc, sh.rpad, d, cs)) != QLORA_OK)
    return st;
  if (counted(launch_convert_bf16(g_acc, sh.m, sh.rpad, sh.rpad, sh.rpad, s, sg, sh.rpad, d.num_sms, cs)) !=
      cudaSuccess)
    return QLORA_ERR_CUDA;

  // 2) XA in fp32: as supplied by the forward, or recomputed
  const float* xa = XA;
  int64_t ld_xa = sh.r;
  if (!xa) {
    CUtensorMap x_k, a_k;
    if (!make_map(&x_k, X, sh.cols, sh.m, sh.cols * 2, 128) ||
        !make_map(&a_k, A, sh.cols, sh.r, sh.cols * 2, 64))
      return QLORA_ERR_CUDA;
    if ((st = run_skinny(false, false, x_k, a_k, sh.m, sh.r, sh.cols, xa_acc, sh.rpad, d, cs)) !=
        QLORA_OK)
      return st;
    xa = xa_acc;
    ld_xa = sh.rpad;
  }

  // 3) dX = dY deq(W) + (s G) A   (fused dequant GEMM, deq(W)^T as the MN-major operand)
  if (dX) {
    const int bn = sh.decode ? 16 : 256;
    CUtensorMap dy_act, sg_map;
    if (!make_map(&dy_act, dY, sh.rows, sh.m, sh.rows * 2, bn) ||
        !make_map(&sg_map, sg, sh.rpad, sh.m, sh.rpad * 2, bn))
      return QLORA_ERR_CUDA;
    FusedArgs fa{};
    fa.codes = W->codes; fa.qabs = W->absmax_q; fa.c2 = W->absmax_c2; fa.mean = W->absmax_mean;
    fa.nw = sh.rows; fa.kw = sh.cols; fa.m = sh.m;
    fa.lora_w = A; fa.r = sh.r; fa.lora_steps = sh.lora_steps;
    fa.ldo = sh.cols; fa.mdim = sh.cols;
    fa.ksteps = static_cast<int>((sh.rows + 63) / 64);
    fa.m_tiles = static_cast<int>((sh.cols + 127) / 128);
    fa.t_tiles = static_cast<int>((sh.m + bn - 1) / bn);
    fa.splits = sh.decode ? choose_splits(fa.m_tiles, fa.ksteps, d.num_sms) : 1;
    fa.m_group = m_group_for(fa.m_tiles, sh.rows);
    fa.out = dX; fa.out_acc = dx_acc;
    fa.cb = codebook_param();
    fa.err = d.err;
    if (fused_timed(FusedDir::kBwd, bn, fa, dy_act, sg_map, d.num_sms, cs) != cudaSuccess)
      return QLORA_ERR_CUDA;
    if (fa.splits > 1 &&
        counted(launch_convert_bf16(dx_acc, sh.m, sh.cols, sh.cols, sh.cols, 1.0f, dX, sh.cols, d.num_sms, cs)) !=
            cudaSuccess)
      return QLORA_ERR_CUDA;
  }

  // 4) LoRA gradients.  Few tokens: fp32 on CUDA cores from the fp32 G and XA.
  if (sh.decode) {
    if (counted(launch_small_grads(g_acc, sh.rpad, xa, ld_xa, X, dY, sh.m, sh.rows, sh.cols, sh.r, s,
                                   dA, dB, d.num_sms, cs)) != cudaSuccess)
      return QLORA_ERR_CUDA;
    return QLORA_OK;
  }
  //    Many tokens: tcgen05 contractions over the tokens with bf16 operands.
  //    dB = dY^T (s XA)  ([rows, r]; both operands MN-major)
  if (counted(launch_convert_bf16(xa, sh.m, sh.r, ld_xa, sh.rpad, s, sxa, sh.rpad, d.num_sms, cs)) != cudaSuccess)
    return QLORA_ERR_CUDA;
  CUtensorMap dy_mn, sxa_mn;
  if (!make_map(&dy_mn, dY, sh.rows, sh.m, sh.rows * 2, 64) ||
      !make_map(&sxa_mn, sxa, sh.rpad, sh.m, sh.rpad * 2, 64))
    return QLORA_ERR_CUDA;
  if ((st = run_skinny(true, true, dy_mn, sxa_mn, sh.rows, sh.r, sh.m, db_acc, sh.rpad, d, cs)) != QLORA_OK)
    return st;
  //    dA^T = X^T (s G)  ([cols, r])
  CUtensorMap x_mn, sg_mn;
  if (!make_map(&x_mn, X, sh.cols, sh.m, sh.cols * 2, 64) ||
      !make_map(&sg_mn, sg, sh.rpad, sh.m, sh.rpad * 2, 64))
    return QLORA_ERR_CUDA;
  if ((st = run_skinny(true, true, x_mn, sg_mn, sh.cols, sh.r, sh.m, da_acc, sh.rpad, d, cs)) != QLORA_OK)
    return st;
  if (counted(launch_convert_f32(db_acc, sh.rows, sh.r, sh.rpad, 1.0f, false, dB, sh.r, d.num_sms, cs)) != cudaSuccess)
    return QLORA_ERR_CUDA;
  if (counted(launch_convert_f32(da_acc, sh.cols, sh.r, sh.rpad, 1.0f, true, dA, sh.cols, d.num_sms, cs)) != cudaSuccess)
    return QLORA_ERR_CUDA;
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
