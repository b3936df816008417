// hstu_attn.cu — host side of libhstu_attn.so: the C ABI declared in include/hstu_attn.h.
//
// Per call: validate arguments on the host -> take a stream-ordered workspace from the
// library's per-device memory pool -> schedule_kernel (work list from seq_offsets /
// num_targets / cached_len) -> hstu_fwd_kernel<d> (persistent, one CTA per SM) -> return the
// workspace on the same stream.  Nothing synchronises; nothing falls back to another path.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <functional>
#include <mutex>
#include <vector>

#include "hstu_attn.h"
#include "hstu_bwd_dq_sm100.cuh"
#include "hstu_bwd_sm100.cuh"
#include "hstu_fwd_sm100.cuh"
#include "gemm_sm100.cuh"
#include "schedule.cuh"

namespace hstu {

// Device error word (kErrBadOffsets | kErrTimeout), one per device context.
__device__ unsigned g_error_word;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
  std::once_flag once;
  cudaError_t init_err = cudaSuccess;
  int num_sms = 0;
  int gemm_clusters = 0;  // resident two-CTA clusters of the two-SM GEMM
  cudaMemPool_t pool = nullptr;
  unsigned* err_word = nullptr;
};
DeviceState g_dev[kMaxDevices];

std::once_flag g_encode_once;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

template <int D>
cudaError_t set_kernel_attrs() {
  cudaError_t e = cudaFuncSetAttribute(hstu_fwd_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       FwdCfg<D>::kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(hstu_fwd_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             FwdCfg<D>::kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(hstu_bwd_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             BwdCfg<D>::kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(hstu_bwd_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             BwdCfg<D>::kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(hstu_bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DqCfg<D>::kSmemBytes);
  return e;
}

// One-time per-device set-up, run with that device current.
void init_device(DeviceState& st, int dev) {
  cudaError_t e = cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) {
    cudaMemPoolProps props;
    std::memset(&props, 0, sizeof(props));
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    e = cudaMemPoolCreate(&st.pool, &props);
  }
  if (e == cudaSuccess) {
    // Keep up to 64 MiB cached between calls so steady-state calls never reach the driver.
    uint64_t keep = 64ull << 20;
    e = cudaMemPoolSetAttribute(st.pool, cudaMemPoolAttrReleaseThreshold, &keep);
  }
  if (e == cudaSuccess) e = cudaGetSymbolAddress(reinterpret_cast<void**>(&st.err_word), g_error_word);
  if (e == cudaSuccess) e = set_kernel_attrs<32>();
  if (e == cudaSuccess) e = set_kernel_attrs<64>();
  if (e == cudaSuccess) e = set_kernel_attrs<128>();
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, GemmCfg::kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_bf16_2sm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Gemm2Cfg::kSmemBytes);
  if (e == cudaSuccess) {
    // How many two-CTA clusters of the two-SM GEMM can be resident at once (SM pairs with room).
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * (st.num_sms / 2));
    cfg.blockDim = dim3(kGemm2Threads);
    cfg.dynamicSmemBytes = Gemm2Cfg::kSmemBytes;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaOccupancyMaxActiveClusters(&st.gemm_clusters, gemm_bf16_2sm_kernel, &cfg);
  }
  st.init_err = e;
}

DeviceState* device_state() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  DeviceState& st = g_dev[dev];
  std::call_once(st.once, init_device, std::ref(st), dev);
  return st.init_err == cudaSuccess ? &st : nullptr;
}

bool encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// 2-D bf16 tensor map over a jagged [rows, H*d] matrix whose rows are `ld` elements apart (ld = 0:
// packed, H*d); box = (box_x columns, 128 rows).
bool encode_rows(CUtensorMap* map, const void* base, int64_t rows, int64_t row_elems, uint32_t box_x,
                 CUtensorMapSwizzle swz, int64_t ld = 0) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_elems), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld > 0 ? ld : row_elems) * 2u};
  cuuint32_t box[2] = {box_x, static_cast<cuuint32_t>(kTileRows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A row-major bf16 [rows, cols] matrix read in boxes of box_rows x 64 columns, 128-byte swizzle.
bool encode_matrix(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, uint32_t box_rows) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2u};
  cuuint32_t box[2] = {64u, box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

// Plan layout (documented in include/hstu_attn.h):
//   int32 header[4] = {work counter, num_items, done counter, 0}
//   int32 q_start[B], padded to 16 bytes
//   int32 block_start[B+1], padded to 16 bytes
//   int4  items[capacity] = {b, block, h, cost}, capacity = H * (total_q / 128 + B)
struct Plan {
  int32_t* counter;
  int32_t* num_items;
  int32_t* done;
  int32_t* q_start;
  int32_t* block_start;
  int4* items;
};

size_t pad16(size_t n_ints) { return ((n_ints * 4 + 15) / 16) * 16; }

int64_t capacity(int32_t B, int32_t H, int32_t total_q) {
  return static_cast<int64_t>(H) * (total_q / kItemRows + B);
}

int64_t plan_bytes(int32_t B, int32_t H, int32_t total_q) {
  return 16 + static_cast<int64_t>(pad16(B) + pad16(static_cast<size_t>(B) + 1)) + capacity(B, H, total_q) * 16;
}

Plan carve(void* base, int32_t B) {
  uint8_t* p = static_cast<uint8_t*>(base);
  Plan w;
  w.counter = reinterpret_cast<int32_t*>(p);
  w.num_items = reinterpret_cast<int32_t*>(p + 4);
  w.done = reinterpret_cast<int32_t*>(p + 8);
  w.q_start = reinterpret_cast<int32_t*>(p + 16);
  w.block_start = reinterpret_cast<int32_t*>(p + 16 + pad16(B));
  w.items = reinterpret_cast<int4*>(p + 16 + pad16(B) + pad16(static_cast<size_t>(B) + 1));
  return w;
}

int cost_bins(int32_t max_seq_len) {
  // A 128-row item computes at most ceil(L/128) + 1 score tiles; the bins leave twice that room.
  int64_t n = 2 * (static_cast<int64_t>(max_seq_len) / kTileRows + 3) + 1;
  return static_cast<int>(n < kMaxCostBins ? n : kMaxCostBins);
}

// Waves a plan's keys need: those the batch's rows can reach, no more than the key space holds (the
// plan kernels clear and scan waves x cost bins keys).
int plan_waves(int64_t rows, int32_t wave_rows, int32_t nbins) {
  const int64_t need = rows > 0 ? (rows + wave_rows - 1) / wave_rows : 1;
  const int64_t fit = nbins > 0 ? kMaxCostBins / nbins : 1;
  const int64_t n = need < fit ? need : fit;
  return static_cast<int>(n > 0 ? n : 1);
}

// Scalar checks shared by every entry point.  Returns HSTU_OK or the status to report.
hstu_status_t check_sizes(int32_t B, int32_t H, int32_t total_kv, int32_t total_q) {
  if (B < 0 || H < 1 || total_kv < 0 || total_q < 0 || total_q > total_kv) return HSTU_ERR_INVALID_ARGUMENT;
  if (capacity(B, H, total_q) > INT_MAX) return HSTU_ERR_UNSUPPORTED;
  return HSTU_OK;
}

hstu_status_t check_tokens(const void* q, const void* k, const void* v, const int32_t* seq_offsets, int32_t H,
                           int32_t d, int32_t total_kv, int32_t total_q, float alpha, float N, const void* out) {
  if (!std::isfinite(alpha) || !std::isfinite(N) || !(N > 0.0f)) return HSTU_ERR_INVALID_ARGUMENT;
  if (d != 32 && d != 64 && d != 128) return HSTU_ERR_UNSUPPORTED;
  const int64_t row_elems = static_cast<int64_t>(H) * d;
  if (row_elems > INT_MAX / 2) return HSTU_ERR_UNSUPPORTED;
  if (total_q == 0) return HSTU_OK;  // nothing is read or written; empty tensors may be NULL
  if (!q || !k || !v || !seq_offsets || !out) return HSTU_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return HSTU_ERR_UNSUPPORTED;
  const size_t qbytes = static_cast<size_t>(total_q) * row_elems * 2;
  const size_t kvbytes = static_cast<size_t>(total_kv) * row_elems * 2;
  if (overlaps(out, qbytes, q, qbytes) || overlaps(out, qbytes, k, kvbytes) || overlaps(out, qbytes, v, kvbytes))
    return HSTU_ERR_INVALID_ARGUMENT;
  return HSTU_OK;
}

cudaError_t launch_plan(const int32_t* seq_offsets, const int32_t* num_targets, const int32_t* cached_len,
                        int32_t B, int32_t H, int32_t total_kv, int32_t total_q, int32_t max_seq_len,
                        const Plan& w, unsigned* err, cudaStream_t stream) {
  SchedArgs a;
  a.seq_offsets = seq_offsets;
  a.num_targets = num_targets;
  a.cached_len = cached_len;
  a.B = B;
  a.H = H;
  a.total_kv = total_kv;
  a.total_q = total_q;
  a.max_seq_len = max_seq_len;
  a.nbins = cost_bins(max_seq_len);
  a.max_items = static_cast<int32_t>(capacity(B, H, total_q));
  // Waves of users whose K and V (sized for d = 128: 512 bytes per row and head) take about a
  // quarter of the 126 MB L2; as many waves as the key space allows.
  a.wave_rows = static_cast<int32_t>((32ll << 20) / (512ll * H) > 0 ? (32ll << 20) / (512ll * H) : 1);
  a.nwaves = plan_waves(total_kv, a.wave_rows, a.nbins);
  a.q_start = w.q_start;
  a.block_start = w.block_start;
  a.items = w.items;
  a.num_items = w.num_items;
  a.work_counter = w.counter;
  a.done_counter = w.done;
  a.err = err;
  schedule_kernel<<<1, kSchedThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

// Launched as a programmatic dependent of the preceding kernel on the stream: its prologue
// (barriers, TMEM allocation, tensor-map prefetch) overlaps the plan kernel, and the producer
// waits for the preceding grid (griddepcontrol.wait) before its first global read.
template <int D, bool kRab>
cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                       int grid, cudaStream_t stream) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kNumThreads);
  cfg.dynamicSmemBytes = FwdCfg<D>::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, hstu_fwd_kernel<D, kRab>, tq, tk, tv, p);
}

// Row strides and the layer epilogue's extra streams for a call whose tensors are column blocks
// of wider matrices (the HSTU layer); every stride 0 means packed [rows, H, d].
struct StridedIO {
  int64_t q_ld = 0, kv_ld = 0, out_ld = 0;
  const void* gate = nullptr;
  int64_t gate_ld = 0;
  void* gate_copy = nullptr;
  void* gate_prod = nullptr;
  uint64_t wait_limit_ns = kWaitLimitNs;
};

// The attention kernel over a plan built for the same offsets.  Arguments already checked.
hstu_status_t launch_attention(DeviceState* st, const void* q, const void* k, const void* v,
                               const int32_t* seq_offsets, const int32_t* num_targets, const int32_t* cached_len,
                               int32_t B, int32_t H, int32_t d, int32_t total_kv, int32_t total_q, float alpha,
                               float N, void* plan, void* out, cudaStream_t stream, const float* rab = nullptr,
                               int32_t rab_len = 0, const StridedIO& io = StridedIO()) {
  if (!encoder()) return HSTU_ERR_CUDA;
  const int64_t row_elems = static_cast<int64_t>(H) * d;
  CUtensorMap tq, tk, tv;
  const uint32_t box_x = d >= 64 ? 64u : 32u;
  const CUtensorMapSwizzle swz = d >= 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (!encode_rows(&tq, q, total_q, row_elems, box_x, swz, io.q_ld) ||
      !encode_rows(&tk, k, total_kv, row_elems, box_x, swz, io.kv_ld) ||
      !encode_rows(&tv, v, total_kv, row_elems, box_x, swz, io.kv_ld))
    return HSTU_ERR_CUDA;
  const Plan w = carve(plan, B);
  FwdParams p;
  p.seq_offsets = seq_offsets;
  p.num_targets = num_targets;
  p.cached_len = cached_len;
  p.q_start = w.q_start;
  p.items = w.items;
  p.num_items = w.num_items;
  p.work_counter = w.counter;
  p.done_counter = w.done;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.out_ld = io.out_ld > 0 ? io.out_ld : row_elems;
  p.gate = static_cast<const __nv_bfloat16*>(io.gate);
  p.gate_ld = io.gate_ld;
  p.gate_copy = static_cast<__nv_bfloat16*>(io.gate_copy);
  p.gate_prod = static_cast<__nv_bfloat16*>(io.gate_prod);
  p.rab = rab;
  p.rab_len = rab_len;
  p.H = H;
  p.half_alpha = 0.5f * alpha;
  p.inv_n = 1.0f / N;
  p.err = st->err_word;
  p.wait_limit_ns = io.wait_limit_ns;
  const int64_t cap = capacity(B, H, total_q);
  const int grid = static_cast<int>(cap < st->num_sms ? cap : st->num_sms);
  cudaError_t e;
  if (rab) {
    if (d == 128) e = launch_fwd<128, true>(tq, tk, tv, p, grid, stream);
    else if (d == 64) e = launch_fwd<64, true>(tq, tk, tv, p, grid, stream);
    else e = launch_fwd<32, true>(tq, tk, tv, p, grid, stream);
  } else {
    if (d == 128) e = launch_fwd<128, false>(tq, tk, tv, p, grid, stream);
    else if (d == 64) e = launch_fwd<64, false>(tq, tk, tv, p, grid, stream);
    else e = launch_fwd<32, false>(tq, tk, tv, p, grid, stream);
  }
  return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

// C = A W^T on the one-SM projection GEMM kernel (128 × 256 tiles).  Arguments already checked.
hstu_status_t launch_gemm_1sm(DeviceState* st, const void* a, const void* w, void* c, int32_t M, int32_t N, int32_t K,
                          cudaStream_t stream) {
  if (!encoder()) return HSTU_ERR_CUDA;
  CUtensorMap ta, tw;
  if (!encode_matrix(&ta, a, M, K, kGemmBM) || !encode_matrix(&tw, w, N, K, kGemmBN)) return HSTU_ERR_CUDA;
  GemmParams p;
  p.c = static_cast<__nv_bfloat16*>(c);
  p.M = M;
  p.N = N;
  p.K = K;
  p.tiles_m = (M + kGemmBM - 1) / kGemmBM;
  p.tiles_n = (N + kGemmBN - 1) / kGemmBN;
  p.err = st->err_word;
  const int64_t ntiles = static_cast<int64_t>(p.tiles_m) * p.tiles_n;
  if (ntiles > INT_MAX) return HSTU_ERR_UNSUPPORTED;
  const int grid = static_cast<int>(ntiles < st->num_sms ? ntiles : st->num_sms);
  // A programmatic dependent of the previous kernel in the stream: its set-up overlaps that kernel's
  // tail, and it waits for it (griddepcontrol.wait) before touching global memory.
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = GemmCfg::kSmemBytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_bf16_kernel, ta, tw, p) == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

// The same product on the two-SM kernel: 256 × 256 tiles, one per cluster of two CTAs.
hstu_status_t launch_gemm_2sm(DeviceState* st, const void* a, const void* w, void* c, int32_t M, int32_t N,
                              int32_t K, cudaStream_t stream) {
  if (!encoder()) return HSTU_ERR_CUDA;
  CUtensorMap ta, tw;
  if (!encode_matrix(&ta, a, M, K, 128) || !encode_matrix(&tw, w, N, K, 128)) return HSTU_ERR_CUDA;
  GemmParams p;
  p.c = static_cast<__nv_bfloat16*>(c);
  p.M = M;
  p.N = N;
  p.K = K;
  p.tiles_m = (M + kGemm2BM - 1) / kGemm2BM;
  p.tiles_n = (N + kGemm2BN - 1) / kGemm2BN;
  p.err = st->err_word;
  const int64_t ntiles = static_cast<int64_t>(p.tiles_m) * p.tiles_n;
  if (ntiles > INT_MAX / 2) return HSTU_ERR_UNSUPPORTED;
  const int clusters = static_cast<int>(ntiles < st->gemm_clusters ? ntiles : st->gemm_clusters);
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // A programmatic dependent of the previous kernel in the stream (as the one-SM launch above).
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(kGemm2Threads);
  cfg.dynamicSmemBytes = Gemm2Cfg::kSmemBytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, gemm_bf16_2sm_kernel, ta, tw, p) == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

// C = A W^T: the two-SM kernel once A has a full 256-row tile, the one-SM kernel below that (or
// when no SM pair can hold a cluster).  Arguments already checked.
hstu_status_t launch_gemm(DeviceState* st, const void* a, const void* w, void* c, int32_t M, int32_t N, int32_t K,
                          cudaStream_t stream) {
  if (M >= kGemm2BM && st->gemm_clusters > 0) return launch_gemm_2sm(st, a, w, c, M, N, K, stream);
  return launch_gemm_1sm(st, a, w, c, M, N, K, stream);
}

// One HSTU layer over a plan built for its offsets (full sequences):
//   UVQK = X W_uvqk^T                     [total, 4D]: blocks U, V, Q, K of D = H d columns
//   A = attention(Q, K, V)                read in place from UVQK; written into CAT[:, D:2D]
//   CAT[:, 0:D] = U, CAT[:, 2D:3D] = U*A  by the attention epilogue
//   Y = CAT W_out^T                       [total, D]
// workspace holds UVQK then CAT.  Arguments already checked.
hstu_status_t run_layer(DeviceState* st, const void* x, const void* w_uvqk, const void* w_out,
                        const int32_t* seq_offsets, const int32_t* num_targets, int32_t B, int32_t H, int32_t d,
                        int32_t total, float alpha, float N, void* plan, void* workspace, void* y,
                        cudaStream_t stream) {
  const int64_t D = static_cast<int64_t>(H) * d;
  auto* uvqk = static_cast<__nv_bfloat16*>(workspace);
  auto* cat = uvqk + static_cast<size_t>(total) * 4 * D;
  hstu_status_t s = launch_gemm(st, x, w_uvqk, uvqk, total, static_cast<int32_t>(4 * D), static_cast<int32_t>(D),
                                stream);
  if (s != HSTU_OK) return s;
  StridedIO io;
  io.q_ld = io.kv_ld = 4 * D;
  io.out_ld = 3 * D;
  io.gate = uvqk;
  io.gate_ld = 4 * D;
  io.gate_copy = cat;
  io.gate_prod = cat + 2 * D;
  s = launch_attention(st, uvqk + 2 * D, uvqk + 3 * D, uvqk + D, seq_offsets, num_targets, nullptr, B, H, d, total,
                       total, alpha, N, plan, cat + D, stream, nullptr, 0, io);
  if (s != HSTU_OK) return s;
  return launch_gemm(st, cat, w_out, y, total, static_cast<int32_t>(D), static_cast<int32_t>(3 * D), stream);
}

// Checks shared by the layer entry points.
hstu_status_t check_layer(const void* x, const void* y, const void* workspace, const int32_t* seq_offsets,
                          int32_t B, int32_t H, int32_t d, int32_t total, float alpha, float N) {
  hstu_status_t s = check_sizes(B, H, total, total);
  if (s != HSTU_OK) return s;
  if (!std::isfinite(alpha) || !std::isfinite(N) || !(N > 0.0f)) return HSTU_ERR_INVALID_ARGUMENT;
  if (d != 32 && d != 64 && d != 128) return HSTU_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(H) * d * 4 > INT_MAX / 2) return HSTU_ERR_UNSUPPORTED;
  if (total == 0 || B == 0) return HSTU_OK;
  if (!x || !y || !workspace || !seq_offsets) return HSTU_ERR_INVALID_ARGUMENT;
  if (!aligned16(x) || !aligned16(y) || !aligned16(workspace)) return HSTU_ERR_UNSUPPORTED;
  return HSTU_OK;
}

int64_t layer_workspace_bytes(int32_t H, int32_t d, int32_t total, int32_t layers) {
  const int64_t D = static_cast<int64_t>(H) * d;
  return static_cast<int64_t>(total) * D * 2 * (7 + (layers > 1 ? 1 : 0));
}

// Plan into a stream-ordered buffer from the library's pool, attention, return the buffer.
hstu_status_t run(const void* q, const void* k, const void* v, const int32_t* seq_offsets,
                  const int32_t* num_targets, const int32_t* cached_len, int32_t B, int32_t H, int32_t d,
                  int32_t total_kv, int32_t total_q, int32_t max_seq_len, float alpha, float N, void* out,
                  void* stream_ptr, const float* rab = nullptr, int32_t rab_len = 0) {
  hstu_status_t s = check_sizes(B, H, total_kv, total_q);
  if (s == HSTU_OK && max_seq_len < 0) s = HSTU_ERR_INVALID_ARGUMENT;
  if (s == HSTU_OK) s = check_tokens(q, k, v, seq_offsets, H, d, total_kv, total_q, alpha, N, out);
  if (s != HSTU_OK) return s;
  if (B == 0 || total_q == 0) return HSTU_OK;
  DeviceState* st = device_state();
  if (!st) return HSTU_ERR_CUDA;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  void* plan = nullptr;
  if (cudaMallocFromPoolAsync(&plan, static_cast<size_t>(plan_bytes(B, H, total_q)), st->pool, stream) !=
      cudaSuccess)
    return HSTU_ERR_CUDA;
  if (launch_plan(seq_offsets, num_targets, cached_len, B, H, total_kv, total_q, max_seq_len, carve(plan, B),
                  st->err_word, stream) != cudaSuccess)
    s = HSTU_ERR_CUDA;
  if (s == HSTU_OK)
    s = launch_attention(st, q, k, v, seq_offsets, num_targets, cached_len, B, H, d, total_kv, total_q, alpha, N,
                         plan, out, stream, rab, rab_len);
  if (cudaFreeAsync(plan, stream) != cudaSuccess && s == HSTU_OK) s = HSTU_ERR_CUDA;
  return s;
}

// Backward plan layout:
//   int32 header[8] = {dq counter, dq items, dq done, 0, kv counter, kv items, kv done, 0}
//   int32 tile_start[B+1], padded to 16 bytes
//   int64 ds_base[B+1], padded to 16 bytes
//   int4  dq_items[cap], kv_items[cap], cap = H * (total / 128 + B)
int64_t bwd_capacity(int32_t B, int32_t H, int32_t total) {
  return static_cast<int64_t>(H) * (total / kTileRows + B);
}

size_t pad16_64(size_t n) { return ((n * 8 + 15) / 16) * 16; }

int64_t bwd_plan_bytes(int32_t B, int32_t H, int32_t total) {
  return 32 + static_cast<int64_t>(pad16(static_cast<size_t>(B) + 1) + pad16_64(static_cast<size_t>(B) + 1)) +
         2 * bwd_capacity(B, H, total) * 16;
}

// dS workspace of the dQ pass, in 128 x 128 tiles: an upper bound on sum over users of
// H * ds_tiles_per_head, from sizes the host knows.  A user of T tiles holds at most
// T (T + 1) / 2 pairs per head, T <= max_seq_len / 128 + 1 and the users' T sum to at most
// total / 128 + B.
int64_t bwd_ds_tiles_bound(int32_t B, int32_t H, int32_t total, int32_t max_seq_len) {
  const int64_t sum_t = static_cast<int64_t>(total) / kTileRows + B;
  const int64_t max_t = static_cast<int64_t>(max_seq_len) / kTileRows + 1;
  return static_cast<int64_t>(H) * (sum_t * (max_t + 1) / 2 + sum_t);
}

constexpr int64_t kDsTileBytes = static_cast<int64_t>(kTileRows) * kTileRows * 2;
std::atomic<uint64_t> g_bwd_ds_limit{16ull << 30};  // bytes; 0: always recompute dS in the dQ pass

// Both backward kernels over a plan written by bwd_schedule_kernel.  Arguments already checked.
template <int D, bool kDQ>
cudaError_t launch_bwd_kernel(const CUtensorMap& f0, const CUtensorMap& f1, const CUtensorMap& s0,
                              const CUtensorMap& s1, const BwdParams& p, int grid, cudaStream_t stream) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kBwdThreads);
  cfg.dynamicSmemBytes = BwdCfg<D>::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, hstu_bwd_kernel<D, kDQ>, f0, f1, s0, s1, p);
}

template <int D>
cudaError_t launch_bwd_dq(const CUtensorMap& tds, const CUtensorMap& tk, const DqParams& p, int grid,
                          cudaStream_t stream) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kDqThreads);
  cfg.dynamicSmemBytes = DqCfg<D>::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, hstu_bwd_dq_kernel<D>, tds, tk, p);
}

// dK/dV, then dQ: from the stored dS tiles when a workspace is given (tds valid), otherwise by
// recomputing S, dP and dS.
template <int D>
cudaError_t launch_bwd_pair(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const CUtensorMap* tds, BwdParams pkv, BwdParams pq,
                            const DqParams& pdq, int grid_kv, int grid_q, cudaStream_t stream) {
  cudaError_t e = launch_bwd_kernel<D, false>(tk, tv, tq, tdo, pkv, grid_kv, stream);
  if (e != cudaSuccess) return e;
  return tds ? launch_bwd_dq<D>(*tds, tk, pdq, grid_q, stream)
             : launch_bwd_kernel<D, true>(tq, tdo, tk, tv, pq, grid_q, stream);
}

hstu_status_t run_bwd(const void* q, const void* k, const void* v, const void* dout, const int32_t* seq_offsets,
                      const int32_t* num_targets, int32_t B, int32_t H, int32_t d, int32_t total,
                      int32_t max_seq_len, float alpha, float N, void* dq, void* dk, void* dv, void* stream_ptr) {
  if (B < 0 || H < 1 || total < 0 || max_seq_len < 0) return HSTU_ERR_INVALID_ARGUMENT;
  if (bwd_capacity(B, H, total) > INT_MAX / 2) return HSTU_ERR_UNSUPPORTED;
  // q, k, v, dq share the checks of a forward call (dq in the role of out), then the other
  // gradients must not overlap any input or each other.
  hstu_status_t s = check_tokens(q, k, v, seq_offsets, H, d, total, total, alpha, N, dq);
  if (s != HSTU_OK) return s;
  if (total == 0 || B == 0) return HSTU_OK;
  if (!dout || !dk || !dv) return HSTU_ERR_INVALID_ARGUMENT;
  if (!aligned16(dout) || !aligned16(dk) || !aligned16(dv)) return HSTU_ERR_UNSUPPORTED;
  const size_t bytes = static_cast<size_t>(total) * H * d * 2;
  const void* ins[4] = {q, k, v, dout};
  void* outs[3] = {dq, dk, dv};
  for (int o = 0; o < 3; ++o) {
    for (int i = 0; i < 4; ++i)
      if (overlaps(outs[o], bytes, ins[i], bytes)) return HSTU_ERR_INVALID_ARGUMENT;
    for (int o2 = o + 1; o2 < 3; ++o2)
      if (overlaps(outs[o], bytes, outs[o2], bytes)) return HSTU_ERR_INVALID_ARGUMENT;
  }
  DeviceState* st = device_state();
  if (!st || !encoder()) return HSTU_ERR_CUDA;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  const int64_t row_elems = static_cast<int64_t>(H) * d;
  CUtensorMap tq, tk, tv, tdo;
  const uint32_t box_x = d >= 64 ? 64u : 32u;
  const CUtensorMapSwizzle swz = d >= 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (!encode_rows(&tq, q, total, row_elems, box_x, swz) || !encode_rows(&tk, k, total, row_elems, box_x, swz) ||
      !encode_rows(&tv, v, total, row_elems, box_x, swz) || !encode_rows(&tdo, dout, total, row_elems, box_x, swz))
    return HSTU_ERR_CUDA;
  void* plan = nullptr;
  if (cudaMallocFromPoolAsync(&plan, static_cast<size_t>(bwd_plan_bytes(B, H, total)), st->pool, stream) !=
      cudaSuccess)
    return HSTU_ERR_CUDA;
  uint8_t* pb = static_cast<uint8_t*>(plan);
  int32_t* header = reinterpret_cast<int32_t*>(pb);
  int32_t* tile_start = reinterpret_cast<int32_t*>(pb + 32);
  long long* ds_base = reinterpret_cast<long long*>(pb + 32 + pad16(static_cast<size_t>(B) + 1));
  const int64_t cap = bwd_capacity(B, H, total);
  int4* dq_items = reinterpret_cast<int4*>(pb + 32 + pad16(static_cast<size_t>(B) + 1) +
                                           pad16_64(static_cast<size_t>(B) + 1));
  int4* kv_items = dq_items + cap;
  // The dS workspace, when its bound fits the limit and the pool has the memory; otherwise the dQ
  // pass recomputes dS.
  const int64_t ds_tiles = bwd_ds_tiles_bound(B, H, total, max_seq_len);
  void* ds_ws = nullptr;
  CUtensorMap tds;
  if (ds_tiles > 0 && ds_tiles * kTileRows <= INT_MAX &&
      static_cast<uint64_t>(ds_tiles * kDsTileBytes) <= g_bwd_ds_limit.load()) {
    if (cudaMallocFromPoolAsync(&ds_ws, static_cast<size_t>(ds_tiles * kDsTileBytes), st->pool, stream) !=
        cudaSuccess) {
      ds_ws = nullptr;
      cudaGetLastError();  // an allocation the pool cannot serve is not an error of the call
    } else if ((reinterpret_cast<uintptr_t>(ds_ws) & 31u) != 0 ||  // the dS stores are 32-byte vectors
               !encode_matrix(&tds, ds_ws, ds_tiles * kTileRows, kTileRows, kTileRows)) {
      cudaFreeAsync(ds_ws, stream);
      ds_ws = nullptr;
    }
  }
  BwdSchedArgs a;
  a.seq_offsets = seq_offsets;
  a.num_targets = num_targets;
  a.B = B;
  a.H = H;
  a.total = total;
  a.max_seq_len = max_seq_len;
  a.nbins = cost_bins(max_seq_len);
  // Waves of users whose streamed pairs (Q and dO, or K and V: 512 bytes per row and head at
  // d = 128) take about a quarter of L2.
  a.wave_rows = static_cast<int32_t>((32ll << 20) / (512ll * H) > 0 ? (32ll << 20) / (512ll * H) : 1);
  a.nwaves = plan_waves(total, a.wave_rows, a.nbins);
  a.max_items = static_cast<int32_t>(cap);
  a.header = header;
  a.tile_start = tile_start;
  a.ds_base = ds_base;
  a.dq_items = dq_items;
  a.kv_items = kv_items;
  a.err = st->err_word;
  bwd_schedule_kernel<<<1, kSchedThreads, 0, stream>>>(a);
  s = cudaGetLastError() == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
  if (s == HSTU_OK) {
    BwdParams pkv;
    pkv.seq_offsets = seq_offsets;
    pkv.num_targets = num_targets;
    pkv.items = kv_items;
    pkv.num_items = header + 5;
    pkv.work_counter = header + 4;
    pkv.done_counter = header + 6;
    pkv.out0 = static_cast<__nv_bfloat16*>(dv);
    pkv.out1 = static_cast<__nv_bfloat16*>(dk);
    pkv.H = H;
    pkv.half_alpha = 0.5f * alpha;
    pkv.ds_scale = 0.5f * alpha / N;
    pkv.inv_n = 1.0f / N;
    pkv.err = st->err_word;
    pkv.ds_ws = static_cast<__nv_bfloat16*>(ds_ws);
    pkv.ds_base = ds_base;
    pkv.ds_cap = ds_ws ? ds_tiles : 0;
    BwdParams pq = pkv;
    pq.ds_ws = nullptr;
    pq.items = dq_items;
    pq.num_items = header + 1;
    pq.work_counter = header + 0;
    pq.done_counter = header + 2;
    pq.out0 = static_cast<__nv_bfloat16*>(dq);
    pq.out1 = nullptr;
    DqParams pdq;
    pdq.seq_offsets = seq_offsets;
    pdq.num_targets = num_targets;
    pdq.items = dq_items;
    pdq.num_items = header + 1;
    pdq.work_counter = header + 0;
    pdq.done_counter = header + 2;
    pdq.ds_base = ds_base;
    pdq.dq = static_cast<__nv_bfloat16*>(dq);
    pdq.H = H;
    pdq.err = st->err_word;
    const CUtensorMap* tdsp = ds_ws ? &tds : nullptr;
    const int grid = static_cast<int>(cap < st->num_sms ? cap : st->num_sms);
    cudaError_t e;
    if (d == 128) e = launch_bwd_pair<128>(tq, tk, tv, tdo, tdsp, pkv, pq, pdq, grid, grid, stream);
    else if (d == 64) e = launch_bwd_pair<64>(tq, tk, tv, tdo, tdsp, pkv, pq, pdq, grid, grid, stream);
    else e = launch_bwd_pair<32>(tq, tk, tv, tdo, tdsp, pkv, pq, pdq, grid, grid, stream);
    if (e != cudaSuccess) s = HSTU_ERR_CUDA;
  }
  if (ds_ws && cudaFreeAsync(ds_ws, stream) != cudaSuccess && s == HSTU_OK) s = HSTU_ERR_CUDA;
  if (cudaFreeAsync(plan, stream) != cudaSuccess && s == HSTU_OK) s = HSTU_ERR_CUDA;
  return s;
}

}  // namespace

// ---------------------------------------------------------------------------------------------
// Allocation-free variant (hstu_attn_fwd_noalloc).  Its plan lives in this fixed device array
// instead of a buffer from the memory pool.  Every device that loads the library holds the
// array until the process exits.  In host code `g_noalloc_plan` names a host-side stand-in, not
// device memory, so the kernels get the device address that cudaGetSymbolAddress returns.
static __device__ __align__(256) unsigned char g_noalloc_plan[HSTU_ATTN_NOALLOC_PLAN_BYTES];

namespace {

struct NoAllocState {
  std::once_flag once;
  cudaError_t err = cudaSuccess;
  DeviceState dev;        // SM count and error word only; its memory pool is never created
  void* plan = nullptr;   // device address of g_noalloc_plan on this device
};
NoAllocState g_noalloc[kMaxDevices];

// Runs once per device, with that device current: looks up the device addresses of the plan
// array and of the error word and sets the kernels' shared-memory limits.  Allocates nothing.
void init_noalloc(NoAllocState& na, int dev) {
  cudaError_t e = cudaDeviceGetAttribute(&na.dev.num_sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) e = cudaGetSymbolAddress(&na.plan, g_noalloc_plan);
  if (e == cudaSuccess) e = cudaGetSymbolAddress(reinterpret_cast<void**>(&na.dev.err_word), g_error_word);
  if (e == cudaSuccess) e = set_kernel_attrs<32>();
  if (e == cudaSuccess) e = set_kernel_attrs<64>();
  if (e == cudaSuccess) e = set_kernel_attrs<128>();
  na.err = e;
}

NoAllocState* noalloc_state() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  NoAllocState& na = g_noalloc[dev];
  std::call_once(na.once, init_noalloc, std::ref(na), dev);
  return na.err == cudaSuccess ? &na : nullptr;
}

}  // namespace
}  // namespace hstu

extern "C" {

hstu_status_t hstu_attn_fwd(const void* q, const void* k, const void* v, const int32_t* seq_offsets,
                            const int32_t* num_targets, int32_t B, int32_t H, int32_t d, int32_t total_tokens,
                            int32_t max_seq_len, float alpha, float N, void* out, void* stream) {
  return hstu::run(q, k, v, seq_offsets, num_targets, nullptr, B, H, d, total_tokens, total_tokens, max_seq_len,
                   alpha, N, out, stream);
}

hstu_status_t hstu_attn_fwd_cached(const void* q, const void* k, const void* v, const int32_t* seq_offsets,
                                   const int32_t* num_targets, const int32_t* cached_len, int32_t B, int32_t H,
                                   int32_t d, int32_t total_kv, int32_t total_q, int32_t max_seq_len, float alpha,
                                   float N, void* out, void* stream) {
  return hstu::run(q, k, v, seq_offsets, num_targets, cached_len, B, H, d, total_kv, total_q, max_seq_len, alpha,
                   N, out, stream);
}

hstu_status_t hstu_attn_fwd_rab(const void* q, const void* k, const void* v, const int32_t* seq_offsets,
                                const int32_t* num_targets, const int32_t* cached_len, const float* rab,
                                int32_t rab_len, int32_t B, int32_t H, int32_t d, int32_t total_kv, int32_t total_q,
                                int32_t max_seq_len, float alpha, float N, void* out, void* stream) {
  if (rab_len < 1 || rab_len > (1 << 24)) return HSTU_ERR_INVALID_ARGUMENT;
  if (!rab && total_q > 0 && B > 0) return HSTU_ERR_INVALID_ARGUMENT;
  if (rab && (reinterpret_cast<uintptr_t>(rab) & 3u)) return HSTU_ERR_UNSUPPORTED;
  return hstu::run(q, k, v, seq_offsets, num_targets, cached_len, B, H, d, total_kv, total_q, max_seq_len, alpha,
                   N, out, stream, rab, rab_len);
}

uint64_t hstu_attn_bwd_workspace_limit(uint64_t max_bytes) { return hstu::g_bwd_ds_limit.exchange(max_bytes); }

hstu_status_t hstu_attn_bwd(const void* q, const void* k, const void* v, const void* dout,
                            const int32_t* seq_offsets, const int32_t* num_targets, int32_t B, int32_t H, int32_t d,
                            int32_t total_tokens, int32_t max_seq_len, float alpha, float N, void* dq, void* dk,
                            void* dv, void* stream) {
  return hstu::run_bwd(q, k, v, dout, seq_offsets, num_targets, B, H, d, total_tokens, max_seq_len, alpha, N, dq,
                       dk, dv, stream);
}

int64_t hstu_attn_plan_bytes(int32_t B, int32_t H, int32_t total_q) {
  if (B < 0 || H < 1 || total_q < 0) return 0;
  return hstu::plan_bytes(B, H, total_q);
}

hstu_status_t hstu_attn_plan(const int32_t* seq_offsets, const int32_t* num_targets, const int32_t* cached_len,
                             int32_t B, int32_t H, int32_t total_kv, int32_t total_q, int32_t max_seq_len,
                             void* plan, int64_t plan_bytes, void* stream_ptr) {
  hstu_status_t s = hstu::check_sizes(B, H, total_kv, total_q);
  if (s != HSTU_OK) return s;
  if (max_seq_len < 0 || !plan || plan_bytes < hstu::plan_bytes(B, H, total_q)) return HSTU_ERR_INVALID_ARGUMENT;
  if (B > 0 && !seq_offsets) return HSTU_ERR_INVALID_ARGUMENT;
  if (!hstu::aligned16(plan)) return HSTU_ERR_UNSUPPORTED;
  hstu::DeviceState* st = hstu::device_state();
  if (!st) return HSTU_ERR_CUDA;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  if (B == 0) return cudaMemsetAsync(plan, 0, 16, stream) == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
  return hstu::launch_plan(seq_offsets, num_targets, cached_len, B, H, total_kv, total_q, max_seq_len,
                           hstu::carve(plan, B), st->err_word, stream) == cudaSuccess
             ? HSTU_OK
             : HSTU_ERR_CUDA;
}

hstu_status_t hstu_attn_fwd_planned(const void* q, const void* k, const void* v, const int32_t* seq_offsets,
                                    const int32_t* num_targets, const int32_t* cached_len, int32_t B, int32_t H,
                                    int32_t d, int32_t total_kv, int32_t total_q, float alpha, float N,
                                    void* plan, void* out, void* stream_ptr) {
  hstu_status_t s = hstu::check_sizes(B, H, total_kv, total_q);
  if (s == HSTU_OK) s = hstu::check_tokens(q, k, v, seq_offsets, H, d, total_kv, total_q, alpha, N, out);
  if (s != HSTU_OK) return s;
  if (B == 0 || total_q == 0) return HSTU_OK;
  if (!plan) return HSTU_ERR_INVALID_ARGUMENT;
  if (!hstu::aligned16(plan)) return HSTU_ERR_UNSUPPORTED;
  hstu::DeviceState* st = hstu::device_state();
  if (!st) return HSTU_ERR_CUDA;
  return hstu::launch_attention(st, q, k, v, seq_offsets, num_targets, cached_len, B, H, d, total_kv, total_q,
                                alpha, N, plan, out, static_cast<cudaStream_t>(stream_ptr));
}

hstu_status_t hstu_attn_get_error(void* stream_ptr) {
  hstu::DeviceState* st = hstu::device_state();
  if (!st) return HSTU_ERR_CUDA;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  unsigned word = 0;
  if (cudaMemcpyAsync(&word, st->err_word, sizeof(word), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return HSTU_ERR_CUDA;
  if (cudaMemsetAsync(st->err_word, 0, sizeof(unsigned), stream) != cudaSuccess) return HSTU_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return HSTU_ERR_CUDA;
  if (word & hstu::kErrTimeout) return HSTU_ERR_TIMEOUT;
  if (word & hstu::kErrBadOffsets) return HSTU_ERR_BAD_OFFSETS;
  return HSTU_OK;
}

hstu_status_t hstu_attn_gemm_bf16(const void* a, const void* w, void* c, int32_t M, int32_t N, int32_t K,
                             void* stream_ptr) {
  if (M < 0 || N < 0 || K <= 0) return HSTU_ERR_INVALID_ARGUMENT;
  if (M == 0 || N == 0) return HSTU_OK;
  if (!a || !w || !c) return HSTU_ERR_INVALID_ARGUMENT;
  if ((K % 8) != 0 || (N % 8) != 0) return HSTU_ERR_UNSUPPORTED;  // 16-byte rows for TMA and stores
  if (!hstu::aligned16(a) || !hstu::aligned16(w) || !hstu::aligned16(c)) return HSTU_ERR_UNSUPPORTED;
  const size_t ca = static_cast<size_t>(M) * K * 2, cw = static_cast<size_t>(N) * K * 2,
               cc = static_cast<size_t>(M) * N * 2;
  if (hstu::overlaps(c, cc, a, ca) || hstu::overlaps(c, cc, w, cw)) return HSTU_ERR_INVALID_ARGUMENT;
  hstu::DeviceState* st = hstu::device_state();
  if (!st) return HSTU_ERR_CUDA;
  return hstu::launch_gemm(st, a, w, c, M, N, K, static_cast<cudaStream_t>(stream_ptr));
}

hstu_status_t hstu_attn_partition(const int32_t* seq_offsets, const int32_t* num_targets,
                                  const int32_t* cached_len, int32_t B, int32_t parts, int32_t* user_start) {
  if (B < 0 || parts < 1 || !user_start || (B > 0 && !seq_offsets)) return HSTU_ERR_INVALID_ARGUMENT;
  // Cost of user b: its visible (query, key) pairs, sum over queried positions i in [c, L) of
  // |A(i)| = i + 1 (history, i < U) or U + 1 (candidate).
  std::vector<int64_t> cost(static_cast<size_t>(B));
  int64_t total = 0, largest = 0;
  for (int32_t b = 0; b < B; ++b) {
    const int64_t L = static_cast<int64_t>(seq_offsets[b + 1]) - seq_offsets[b];
    const int64_t T = num_targets ? num_targets[b] : 0;
    const int64_t c = cached_len ? cached_len[b] : 0;
    if (L < 0 || T < 0 || T > L || c < 0 || c > L - T) return HSTU_ERR_BAD_OFFSETS;
    const int64_t U = L - T;
    const int64_t hist = c < U ? (U * (U + 1) - c * (c + 1)) / 2 : 0;
    cost[b] = hist + (L - (U > c ? U : c)) * (U + 1);
    total += cost[b];
    largest = cost[b] > largest ? cost[b] : largest;
  }
  // Smallest cap such that consecutive users fill at most `parts` parts of cost <= cap.
  auto parts_needed = [&](int64_t cap) {
    int32_t n = 1;
    int64_t run = 0;
    for (int32_t b = 0; b < B; ++b) {
      if (run + cost[b] > cap) {
        ++n;
        run = 0;
      }
      run += cost[b];
    }
    return n;
  };
  int64_t lo = largest, hi = total > largest ? total : largest;
  while (lo < hi) {
    const int64_t mid = lo + (hi - lo) / 2;
    if (parts_needed(mid) <= parts) hi = mid;
    else lo = mid + 1;
  }
  // Fill parts left to right under that cap; parts left over at the end are empty.
  int32_t part = 0;
  int64_t run = 0;
  user_start[0] = 0;
  for (int32_t b = 0; b < B; ++b) {
    if (run + cost[b] > lo && run > 0 && part + 1 < parts) {
      user_start[++part] = b;
      run = 0;
    }
    run += cost[b];
  }
  for (int32_t k = part + 1; k <= parts; ++k) user_start[k] = B;
  return HSTU_OK;
}

int64_t hstu_layer_workspace_bytes(int32_t H, int32_t d, int32_t total, int32_t num_layers) {
  if (H < 1 || d < 1 || total < 0 || num_layers < 1) return 0;
  return hstu::layer_workspace_bytes(H, d, total, num_layers);
}

hstu_status_t hstu_layer_fwd(const void* x, const void* w_uvqk, const void* w_out, const int32_t* seq_offsets,
                             const int32_t* num_targets, int32_t B, int32_t H, int32_t d, int32_t total,
                             float alpha, float N, void* plan, void* workspace, int64_t workspace_bytes, void* y,
                             void* stream_ptr) {
  hstu_status_t s = hstu::check_layer(x, y, workspace, seq_offsets, B, H, d, total, alpha, N);
  if (s != HSTU_OK || total == 0 || B == 0) return s;
  if (!w_uvqk || !w_out || !plan) return HSTU_ERR_INVALID_ARGUMENT;
  if (!hstu::aligned16(w_uvqk) || !hstu::aligned16(w_out) || !hstu::aligned16(plan)) return HSTU_ERR_UNSUPPORTED;
  if (workspace_bytes < hstu::layer_workspace_bytes(H, d, total, 1)) return HSTU_ERR_INVALID_ARGUMENT;
  const size_t act = static_cast<size_t>(total) * H * d * 2;
  if (hstu::overlaps(y, act, workspace, static_cast<size_t>(workspace_bytes)) ||
      hstu::overlaps(x, act, workspace, static_cast<size_t>(workspace_bytes)))
    return HSTU_ERR_INVALID_ARGUMENT;
  hstu::DeviceState* st = hstu::device_state();
  if (!st) return HSTU_ERR_CUDA;
  return hstu::run_layer(st, x, w_uvqk, w_out, seq_offsets, num_targets, B, H, d, total, alpha, N, plan, workspace,
                         y, static_cast<cudaStream_t>(stream_ptr));
}

hstu_status_t hstu_layers_fwd(int32_t num_layers, const void* x, const void* const* w_uvqk,
                              const void* const* w_out, const int32_t* seq_offsets, const int32_t* num_targets,
                              int32_t B, int32_t H, int32_t d, int32_t total, int32_t max_seq_len, float alpha,
                              float N, void* workspace, int64_t workspace_bytes, void* y, void* stream_ptr) {
  if (num_layers < 1 || !w_uvqk || !w_out || max_seq_len < 0) return HSTU_ERR_INVALID_ARGUMENT;
  hstu_status_t s = hstu::check_layer(x, y, workspace, seq_offsets, B, H, d, total, alpha, N);
  if (s != HSTU_OK || total == 0 || B == 0) return s;
  for (int32_t l = 0; l < num_layers; ++l) {
    if (!w_uvqk[l] || !w_out[l]) return HSTU_ERR_INVALID_ARGUMENT;
    if (!hstu::aligned16(w_uvqk[l]) || !hstu::aligned16(w_out[l])) return HSTU_ERR_UNSUPPORTED;
  }
  if (workspace_bytes < hstu::layer_workspace_bytes(H, d, total, num_layers)) return HSTU_ERR_INVALID_ARGUMENT;
  const size_t act = static_cast<size_t>(total) * H * d * 2;
  if (hstu::overlaps(y, act, workspace, static_cast<size_t>(workspace_bytes)) ||
      hstu::overlaps(x, act, workspace, static_cast<size_t>(workspace_bytes)))
    return HSTU_ERR_INVALID_ARGUMENT;
  hstu::DeviceState* st = hstu::device_state();
  if (!st) return HSTU_ERR_CUDA;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  // One plan for every layer: the jagged structure does not change between layers.
  void* plan = nullptr;
  if (cudaMallocFromPoolAsync(&plan, static_cast<size_t>(hstu::plan_bytes(B, H, total)), st->pool, stream) !=
      cudaSuccess)
    return HSTU_ERR_CUDA;
  if (hstu::launch_plan(seq_offsets, num_targets, nullptr, B, H, total, total, max_seq_len, hstu::carve(plan, B),
                        st->err_word, stream) != cudaSuccess)
    s = HSTU_ERR_CUDA;
  // Layer l reads its input (x, then the hidden buffer after UVQK and CAT) and writes its output
  // (y for the last layer); a layer's input is dead once its first projection has run, so the
  // hidden buffer can be read and rewritten by the same layer.
  auto* hidden = static_cast<uint8_t*>(workspace) + static_cast<size_t>(total) * H * d * 2 * 7;
  for (int32_t l = 0; l < num_layers && s == HSTU_OK; ++l) {
    const void* in = l == 0 ? x : hidden;
    void* out = l == num_layers - 1 ? y : hidden;
    s = hstu::run_layer(st, in, w_uvqk[l], w_out[l], seq_offsets, num_targets, B, H, d, total, alpha, N, plan,
                        workspace, out, stream);
  }
  if (cudaFreeAsync(plan, stream) != cudaSuccess && s == HSTU_OK) s = HSTU_ERR_CUDA;
  return s;
}

hstu_status_t hstu_attn_selfcheck_wait_timeout(uint64_t limit_ns, void* stream_ptr) {
  if (limit_ns == 0 || limit_ns > 1000000000ull) return HSTU_ERR_INVALID_ARGUMENT;
  hstu::DeviceState* st = hstu::device_state();
  if (!st) return HSTU_ERR_CUDA;
  hstu::wait_timeout_selfcheck_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream_ptr)>>>(st->err_word, limit_ns);
  return cudaGetLastError() == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

hstu_status_t hstu_attn_selfcheck_fwd_timeout(const void* q, const void* k, const void* v,
                                              const int32_t* seq_offsets, const int32_t* num_targets, int32_t B,
                                              int32_t H, int32_t d, int32_t total_tokens, int32_t max_seq_len,
                                              float alpha, float N, void* out, uint64_t limit_ns, void* stream_ptr) {
  if (limit_ns == 0 || limit_ns > 1000000000ull) return HSTU_ERR_INVALID_ARGUMENT;
  hstu_status_t s = hstu::check_sizes(B, H, total_tokens, total_tokens);
  if (s == HSTU_OK && max_seq_len < 0) s = HSTU_ERR_INVALID_ARGUMENT;
  if (s == HSTU_OK) s = hstu::check_tokens(q, k, v, seq_offsets, H, d, total_tokens, total_tokens, alpha, N, out);
  if (s != HSTU_OK || B == 0 || total_tokens == 0) return s;
  hstu::DeviceState* st = hstu::device_state();
  if (!st) return HSTU_ERR_CUDA;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  void* plan = nullptr;
  if (cudaMallocFromPoolAsync(&plan, static_cast<size_t>(hstu::plan_bytes(B, H, total_tokens)), st->pool, stream) !=
      cudaSuccess)
    return HSTU_ERR_CUDA;
  if (hstu::launch_plan(seq_offsets, num_targets, nullptr, B, H, total_tokens, total_tokens, max_seq_len,
                        hstu::carve(plan, B), st->err_word, stream) != cudaSuccess)
    s = HSTU_ERR_CUDA;
  hstu::StridedIO io;
  io.wait_limit_ns = limit_ns;
  if (s == HSTU_OK)
    s = hstu::launch_attention(st, q, k, v, seq_offsets, num_targets, nullptr, B, H, d, total_tokens, total_tokens,
                               alpha, N, plan, out, stream, nullptr, 0, io);
  if (cudaFreeAsync(plan, stream) != cudaSuccess && s == HSTU_OK) s = HSTU_ERR_CUDA;
  return s;
}

const char* hstu_attn_status_string(hstu_status_t s) {
  switch (s) {
    case HSTU_OK: return "HSTU_OK";
    case HSTU_ERR_INVALID_ARGUMENT: return "HSTU_ERR_INVALID_ARGUMENT";
    case HSTU_ERR_UNSUPPORTED: return "HSTU_ERR_UNSUPPORTED";
    case HSTU_ERR_CUDA: return "HSTU_ERR_CUDA";
    case HSTU_ERR_BAD_OFFSETS: return "HSTU_ERR_BAD_OFFSETS";
    case HSTU_ERR_TIMEOUT: return "HSTU_ERR_TIMEOUT";
  }
  return "HSTU_ERR_UNKNOWN";
}

hstu_status_t hstu_attn_fwd_noalloc(const void* q, const void* k, const void* v, const int32_t* seq_offsets,
                                    const int32_t* num_targets, const int32_t* cached_len, int32_t B, int32_t H,
                                    int32_t d, int32_t total_kv, int32_t total_q, int32_t max_seq_len, float alpha,
                                    float N, void* out, void* stream_ptr) {
  hstu_status_t s = hstu::check_sizes(B, H, total_kv, total_q);
  if (s == HSTU_OK && max_seq_len < 0) s = HSTU_ERR_INVALID_ARGUMENT;
  if (s == HSTU_OK) s = hstu::check_tokens(q, k, v, seq_offsets, H, d, total_kv, total_q, alpha, N, out);
  if (s != HSTU_OK) return s;
  if (hstu::plan_bytes(B, H, total_q) > static_cast<int64_t>(HSTU_ATTN_NOALLOC_PLAN_BYTES))
    return HSTU_ERR_UNSUPPORTED;  // the batch needs a bigger plan than the fixed array holds
  if (B == 0 || total_q == 0) return HSTU_OK;
  hstu::NoAllocState* na = hstu::noalloc_state();
  if (!na) return HSTU_ERR_CUDA;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  // The plan kernel rewrites every plan word the attention kernel reads (header counters
  // included), so what an earlier call left in the array does not matter.
  if (hstu::launch_plan(seq_offsets, num_targets, cached_len, B, H, total_kv, total_q, max_seq_len,
                        hstu::carve(na->plan, B), na->dev.err_word, stream) != cudaSuccess)
    return HSTU_ERR_CUDA;
  return hstu::launch_attention(&na->dev, q, k, v, seq_offsets, num_targets, cached_len, B, H, d, total_kv,
                                total_q, alpha, N, na->plan, out, stream);
}

}  // extern "C"
