// api.cu -- the C ABI of the library (include/seer.h): argument validation,
// workspace carving, TMA tensor-map encoding and kernel launches.  Every call
// is asynchronous on the caller's stream; nothing here allocates device
// memory.
#include <cmath>
#include <cstdint>
#include <vector>
#include <cstring>
#include <mutex>
#include <new>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/seer.h"
#include "attn.cuh"
#include "blockmax.cuh"
#include "fwd.cuh"
#include "gate_train.cuh"
#include "decode.cuh"
#include "attn_tf32.cuh"
#include "common.cuh"
#include "gate.cuh"
#include "ptx.cuh"

namespace {

thread_local int32_t g_last_cuda_error = 0;
// seer_testing_attn_wait_fault's settings for this host thread
thread_local int32_t g_test_skip_qk_commit = -1;
thread_local unsigned long long g_test_wait_limit_ns = 0;

seer_status cuda_fail(cudaError_t e) {
  g_last_cuda_error = (int32_t)e;
  return SEER_ERR_CUDA;
}

#define SEER_CUDA(x)                            \
  do {                                          \
    cudaError_t e_ = (x);                       \
    if (e_ != cudaSuccess) return cuda_fail(e_); \
  } while (0)

bool dims_ok(const seer_dims* d) {
  if (!d) return false;
  if (d->B < 1 || d->Hq < 1 || d->Hkv < 1 || d->n < 1) return false;
  if (d->Hq % d->Hkv != 0) return false;
  if (d->n % seer::kBlock != 0) return false;
  // TMA row coordinates and the persistent work index are 32-bit
  if ((long long)d->B * d->Hq * d->n >= (1LL << 31)) return false;
  return true;
}

seer_status dims_supported(const seer_dims* d) {
  if (d->block != seer::kBlock) return SEER_ERR_UNSUPPORTED;
  if (d->d != 64 && d->d != 128) return SEER_ERR_UNSUPPORTED;
  return SEER_OK;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// dependency on libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)f;
  });
  return fn;
}

// 2-D bf16 map over [rows, d] with a (64 x box_rows) box, 128-byte swizzle.
bool make_tmap(CUtensorMap* tm, const void* base, long long rows, int d, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D fp32 map over [rows, d] with a 32 x 64 box (128 bytes by 64 rows),
// 128-byte swizzle.
bool make_tmap_f32(CUtensorMap* tm, const void* base, long long rows, int d, int box_rows = 64) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 4};
  cuuint32_t box[2] = {32, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D fp32 map that reads a [rows, inner] tensor as panels: x = 32 floats
// of a row (128 bytes), y = rows, z = the row's 32-float chunks (128 bytes
// apart).  One box {32, box_rows, inner / 32} lands in shared memory as
// inner/32 panels of box_rows x 128 bytes, 128-byte swizzled: a whole tile
// per copy.
bool make_tmap_f32_panels(CUtensorMap* tm, const void* base, long long rows, int inner, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {32, (cuuint64_t)rows, (cuuint64_t)(inner / 32)};
  cuuint64_t strides[2] = {(cuuint64_t)inner * 4, 128};
  cuuint32_t box[3] = {32, (cuuint32_t)box_rows, (cuuint32_t)(inner / 32)};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D fp32 map over a batch of row-major matrices C[z][rows][cols] with row
// stride ld and batch stride bs (in elements): a box of 32 columns x 128 rows
// x 1 matrix, 128-byte swizzle (the TMA-store staging layout).
bool make_tmap_f32_batched(CUtensorMap* tm, const void* base, int cols, int rows, int batch, long long ld,
                           long long bs) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)batch};
  cuuint64_t strides[2] = {(cuuint64_t)ld * 4, (cuuint64_t)bs * 4};
  cuuint32_t box[3] = {32, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 map over a row-major [rows, inner] matrix seen as (64 columns,
// rows, inner/64 panels): a box of 64 x box_rows x inner/64 lands as
// inner/64 consecutive 128-byte-swizzled panels of box_rows rows.
bool make_tmap_bf16_panels(CUtensorMap* tm, const void* base, long long rows, int inner, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)rows, (cuuint64_t)(inner / 64)};
  cuuint64_t strides[2] = {(cuuint64_t)inner * 2, 128};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, (cuuint32_t)(inner / 64)};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 map over [rows, 64] (128-byte rows) with a box of box_rows rows.
bool make_tmap_rows(CUtensorMap* tm, const void* base, long long rows, int box_rows) {
  return make_tmap(tm, base, rows, 64, box_rows);
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

constexpr unsigned long long kTimeoutNs = 2000000000ull;  // 2 s per bounded wait
// header word of seer_sparse_attn's dense / sparse choice (1: not the all-ones mask)
constexpr int kWsNotDenseWord = 40;

__global__ void f32_to_bf16_kernel(const float* __restrict__ x, __nv_bfloat16* __restrict__ y,
                                   long long n) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    y[i] = __float2bfloat16_rn(x[i]);
}

cudaError_t to_bf16(const void* x, void* y, long long n, cudaStream_t st) {
  f32_to_bf16_kernel<<<1184, 256, 0, st>>>((const float*)x, (__nv_bfloat16*)y, n);
  return cudaGetLastError();
}

struct GateWs {
  size_t qbar, kbar, qt, kt, logits, qlo, klo, qbar_hi, qbar_lo, kbar_hi, kbar_lo, wq_hi, wq_lo, wk_hi, wk_lo, total;
};

// The causal logits run on the tensor cores (three tf32 products) when the
// gate hidden size is a multiple of 32; otherwise on the fp32 SIMT GEMM.
bool gate_tf32x3(int h) { return h % 32 == 0; }
// The projections too, when the head dimension is a multiple of 32 as well.
bool gate_proj_tf32x3(int h, int d) { return h % 32 == 0 && d % 32 == 0; }

GateWs gate_ws(const seer_dims* d, int h) {
  const long long nb = d->n / seer::kBlock;
  seer::WsCarver c;
  GateWs w;
  w.qbar = c.take(sizeof(float) * d->B * d->Hq * nb * d->d);
  w.kbar = c.take(sizeof(float) * d->B * d->Hkv * nb * 3 * d->d);
  w.qt = c.take(sizeof(float) * d->B * d->Hq * nb * h);
  w.kt = c.take(sizeof(float) * d->B * d->Hkv * nb * h);
  w.logits = c.take(sizeof(float) * d->B * d->Hq * nb * nb);
  // tf32 remainders of q~ and k~ (the tensor-core logits only)
  w.qlo = gate_tf32x3(h) ? c.take(sizeof(float) * d->B * d->Hq * nb * h) : 0;
  w.klo = gate_tf32x3(h) ? c.take(sizeof(float) * d->B * d->Hkv * nb * h) : 0;
  // tf32 parts of the pooled Q / K and of the weights, for the projections
  // (the pooled fp32 values stay as they are: the distillation step reads them)
  const bool pj = gate_proj_tf32x3(h, d->d);
  w.qbar_hi = pj ? c.take(sizeof(float) * d->B * d->Hq * nb * d->d) : 0;
  w.qbar_lo = pj ? c.take(sizeof(float) * d->B * d->Hq * nb * d->d) : 0;
  w.kbar_hi = pj ? c.take(sizeof(float) * d->B * d->Hkv * nb * 3 * d->d) : 0;
  w.kbar_lo = pj ? c.take(sizeof(float) * d->B * d->Hkv * nb * 3 * d->d) : 0;
  w.wq_hi = pj ? c.take(sizeof(float) * d->Hq * h * d->d) : 0;
  w.wq_lo = pj ? c.take(sizeof(float) * d->Hq * h * d->d) : 0;
  w.wk_hi = pj ? c.take(sizeof(float) * d->Hkv * h * 3 * d->d) : 0;
  w.wk_lo = pj ? c.take(sizeof(float) * d->Hkv * h * 3 * d->d) : 0;
  w.total = c.off;
  return w;
}

// The gate's workspace, then the KL step's: per-row loss terms and the
// gradients of q~ and k~ (dz is written over the logits).
struct GateTrainWs {
  GateWs gate;
  size_t row_loss, dqt, dkt, total;
};

GateTrainWs gate_train_ws(const seer_dims* d, int h) {
  const long long nb = d->n / seer::kBlock;
  GateTrainWs w;
  w.gate = gate_ws(d, h);
  seer::WsCarver c;
  c.off = w.gate.total;
  w.row_loss = c.take(sizeof(float) * d->B * d->Hq * nb);
  w.dqt = c.take(sizeof(float) * d->B * d->Hq * nb * h);
  w.dkt = c.take(sizeof(float) * d->B * d->Hkv * nb * h);
  w.total = c.off;
  return w;
}

struct AttnWs {
  size_t q16, v16, kt, redo, total;
};

// fp32 Q and V converted to bf16 (fp32 inputs only; bf16 V is read in
// place), then the K^T block records (B * Hkv * n * d bf16: d rows x 64 keys
// per 64-key block).
AttnWs attn_ws(const seer_dims* d, seer_dtype dt) {
  seer::WsCarver c;
  AttnWs w{0, 0, 0, 0, 0};
  if (dt == SEER_FP32) {
    w.q16 = c.take(2ull * d->B * d->Hq * d->n * d->d);
    w.v16 = c.take(2ull * d->B * d->Hkv * d->n * d->d);
  }
  w.kt = c.take(2ull * d->B * d->Hkv * d->n * d->d);
  // units flagged for the exact fallback (one int32 per unit at most)
  w.redo = c.take(sizeof(int32_t) * (size_t)d->B * d->Hq * (d->n / seer::kBlock));
  w.total = c.off;
  return w;
}

struct BmaxWs {
  size_t q16, k16, r, total;
  int ctas;
};

BmaxWs bmax_ws(const seer_dims* d, seer_dtype dt, int sms) {
  seer::WsCarver c;
  BmaxWs w{0, 0, 0, 0, 0};
  if (dt == SEER_FP32) {
    w.q16 = c.take(2ull * d->B * d->Hq * d->n * d->d);
    w.k16 = c.take(2ull * d->B * d->Hkv * d->n * d->d);
  }
  const long long nb = d->n / seer::kBlock;
  w.ctas = sms;
  w.r = c.take(sizeof(float) * (size_t)sms * 256 * nb);  // [ctas][nb][2 column halves][128 rows]
  w.total = c.off;
  return w;
}

seer_status begin_ws(void* ws, size_t ws_bytes, size_t need, cudaStream_t st) {
  if (!ws || !aligned(ws, 256) || ws_bytes < need) return SEER_ERR_WORKSPACE;
  SEER_CUDA(cudaMemsetAsync(ws, 0, sizeof(seer::WsHeader), st));
  return SEER_OK;
}

}  // namespace

namespace seer {
void set_last_cuda_error(int32_t e) { g_last_cuda_error = e; }
}  // namespace seer

extern "C" {

const char* seer_version(void) { return "0.1.0"; }

int32_t seer_last_cuda_error(void) { return g_last_cuda_error; }

void seer_testing_attn_wait_fault(int32_t step, uint64_t wait_limit_ns) {
  g_test_skip_qk_commit = step < 0 ? -1 : step;
  g_test_wait_limit_ns = wait_limit_ns;
}

const char* seer_status_string(seer_status s) {
  switch (s) {
    case SEER_OK: return "SEER_OK";
    case SEER_ERR_INVALID_ARG: return "SEER_ERR_INVALID_ARG";
    case SEER_ERR_UNSUPPORTED: return "SEER_ERR_UNSUPPORTED";
    case SEER_ERR_CAPACITY: return "SEER_ERR_CAPACITY";
    case SEER_ERR_CUDA: return "SEER_ERR_CUDA";
    case SEER_ERR_TIMEOUT: return "SEER_ERR_TIMEOUT";
    case SEER_ERR_DEVICE_CHECK: return "SEER_ERR_DEVICE_CHECK";
    case SEER_ERR_WORKSPACE: return "SEER_ERR_WORKSPACE";
  }
  return "SEER_ERR_UNKNOWN";
}

seer_status seer_workspace_status(const void* ws, seer_stream_t stream) {
  if (!ws) return SEER_ERR_WORKSPACE;
  uint32_t h[2] = {0, 0};
  cudaStream_t st = (cudaStream_t)stream;
  SEER_CUDA(cudaMemcpyAsync(h, ws, sizeof(h), cudaMemcpyDeviceToHost, st));
  SEER_CUDA(cudaStreamSynchronize(st));
  switch (h[0]) {
    case seer::kDevOk: return SEER_OK;
    case seer::kDevTimeout: return SEER_ERR_TIMEOUT;
    default: return SEER_ERR_DEVICE_CHECK;
  }
}

// ------------------------------------------------------------------- gate --
size_t seer_gate_workspace_size(const seer_dims* dims, int32_t h) {
  if (!dims_ok(dims) || h < 1) return 0;
  return gate_ws(dims, h).total;
}

size_t seer_gate_kl_backward_workspace_size(const seer_dims* dims, int32_t h) {
  if (!dims_ok(dims) || h < 1) return 0;
  return gate_train_ws(dims, h).total;
}

seer_status seer_gate_kl_backward(const seer_dims* dims, const void* Q, const void* K, seer_dtype dtype,
                                  const float* Wq, const float* Wk, int32_t h, const float* gt, float* loss,
                                  float* dWq, float* dWk, void* ws, size_t ws_bytes, seer_stream_t stream) {
  if (!dims_ok(dims) || !Q || !K || !Wq || !Wk || !gt || !loss || !dWq || !dWk) return SEER_ERR_INVALID_ARG;
  if (dtype != SEER_BF16 && dtype != SEER_FP32) return SEER_ERR_INVALID_ARG;
  if (h < 1 || h > 256 || (h % 4) != 0) return SEER_ERR_INVALID_ARG;
  seer_status s = dims_supported(dims);
  if (s != SEER_OK) return s;
  if (!aligned(Q, 16) || !aligned(K, 16)) return SEER_ERR_INVALID_ARG;
  const GateTrainWs w = gate_train_ws(dims, h);
  cudaStream_t st = (cudaStream_t)stream;
  s = begin_ws(ws, ws_bytes, w.total, st);
  if (s != SEER_OK) return s;

  uint8_t* base = (uint8_t*)ws;
  float* qbar = (float*)(base + w.gate.qbar);
  float* kbar = (float*)(base + w.gate.kbar);
  float* qt = (float*)(base + w.gate.qt);
  float* kt = (float*)(base + w.gate.kt);
  float* zdz = (float*)(base + w.gate.logits);
  float* row_loss = (float*)(base + w.row_loss);
  float* dqt = (float*)(base + w.dqt);
  float* dkt = (float*)(base + w.dkt);
  const int B = dims->B, Hq = dims->Hq, Hkv = dims->Hkv, n = dims->n, d = dims->d;
  const int nb = n / seer::kBlock, G = Hq / Hkv;
  const float inv_sqrt_d = (float)(1.0 / std::sqrt((double)d));
  const long long rows = (long long)B * Hq * nb;

  // gate forward, as in seer_gate (no RoPE): pooling, projections, logits
  SEER_CUDA(seer::launch_pool(Q, dtype, false, (long long)B * Hq, n, d, qbar, st));
  SEER_CUDA(seer::launch_pool(K, dtype, true, (long long)B * Hkv, n, d, kbar, st));
  SEER_CUDA(seer::launch_gemm_nt(qbar, Wq, qt, nb, h, d, (long long)nb * d, (long long)h * d,
                                 (long long)nb * h, h, B * Hq, Hq, 0, 1, 1.0f, false, st));
  SEER_CUDA(seer::launch_gemm_nt(kbar, Wk, kt, nb, h, 3 * d, (long long)nb * 3 * d,
                                 (long long)h * 3 * d, (long long)nb * h, h, B * Hkv, Hkv, 0, 1,
                                 1.0f, false, st));
  SEER_CUDA(seer::launch_gemm_nt(qt, kt, zdz, nb, nb, h, (long long)nb * h, (long long)nb * h,
                                 (long long)nb * nb, nb, B * Hq, Hq, Hkv, G, inv_sqrt_d, true, st));
  // KL per row and dz over the logits, then the loss
  SEER_CUDA(seer::launch_kl_rows(zdz, gt, row_loss, rows, nb, st));
  SEER_CUDA(seer::launch_loss_sum(row_loss, rows, loss, st));
  seer::GemmBatched g{};
  // dq~[b,hq] = dz[b,hq] k~[b,g] / sqrt(d): (i, j) x (j, c); dz is zero for j > i
  g = seer::GemmBatched{};
  g.A = zdz; g.B = kt; g.C = dqt;
  g.M = nb; g.N = h; g.K = nb; g.R = 1; g.Z1 = B; g.Z2 = Hq; g.b_div = G; g.band = 1;
  g.a_m = nb; g.a_k = 1; g.a_z1 = (long long)Hq * nb * nb; g.a_z2 = (long long)nb * nb; g.a_r = 0;
  g.b_k = h; g.b_n = 1; g.b_z1 = (long long)Hkv * nb * h; g.b_z2 = (long long)nb * h; g.b_r = 0;
  g.c_m = h; g.c_n = 1; g.c_z1 = (long long)Hq * nb * h; g.c_z2 = (long long)nb * h;
  g.alpha = inv_sqrt_d;
  SEER_CUDA(seer::launch_gemm_batched(g, st));
  // dk~[b,g] = sum over the G query heads of dz^T q~ / sqrt(d): (j, i) x (i, c); nonzero for i >= j
  g = seer::GemmBatched{};
  g.A = zdz; g.B = qt; g.C = dkt;
  g.M = nb; g.N = h; g.K = nb; g.R = G; g.Z1 = B; g.Z2 = Hkv; g.b_div = 1; g.band = 2;
  g.a_m = 1; g.a_k = nb; g.a_z1 = (long long)Hq * nb * nb; g.a_z2 = (long long)G * nb * nb;
  g.a_r = (long long)nb * nb;
  g.b_k = h; g.b_n = 1; g.b_z1 = (long long)Hq * nb * h; g.b_z2 = (long long)G * nb * h; g.b_r = (long long)nb * h;
  g.c_m = h; g.c_n = 1; g.c_z1 = (long long)Hkv * nb * h; g.c_z2 = (long long)nb * h;
  g.alpha = inv_sqrt_d;
  SEER_CUDA(seer::launch_gemm_batched(g, st));
  // dWq[hq] = sum_b dq~[b,hq]^T qbar[b,hq]: (c, i) x (i, e)
  g = seer::GemmBatched{};
  g.A = dqt; g.B = qbar; g.C = dWq;
  g.M = h; g.N = d; g.K = nb; g.R = B; g.Z1 = 1; g.Z2 = Hq; g.b_div = 1; g.band = 0;
  g.a_m = 1; g.a_k = h; g.a_z1 = 0; g.a_z2 = (long long)nb * h; g.a_r = (long long)Hq * nb * h;
  g.b_k = d; g.b_n = 1; g.b_z1 = 0; g.b_z2 = (long long)nb * d; g.b_r = (long long)Hq * nb * d;
  g.c_m = d; g.c_n = 1; g.c_z1 = 0; g.c_z2 = (long long)h * d;
  g.alpha = 1.0f;
  SEER_CUDA(seer::launch_gemm_batched(g, st));
  // dWk[g] = sum_b dk~[b,g]^T kbar[b,g]: (c, j) x (j, e)
  g = seer::GemmBatched{};
  g.A = dkt; g.B = kbar; g.C = dWk;
  g.M = h; g.N = 3 * d; g.K = nb; g.R = B; g.Z1 = 1; g.Z2 = Hkv; g.b_div = 1; g.band = 0;
  g.a_m = 1; g.a_k = h; g.a_z1 = 0; g.a_z2 = (long long)nb * h; g.a_r = (long long)Hkv * nb * h;
  g.b_k = 3 * d; g.b_n = 1; g.b_z1 = 0; g.b_z2 = (long long)nb * 3 * d; g.b_r = (long long)Hkv * nb * 3 * d;
  g.c_m = 3 * d; g.c_n = 1; g.c_z1 = 0; g.c_z2 = (long long)h * 3 * d;
  g.alpha = 1.0f;
  SEER_CUDA(seer::launch_gemm_batched(g, st));
  return SEER_OK;
}

int32_t seer_gate_required_cap(const seer_dims* dims, seer_select_mode mode, int32_t k,
                               float density) {
  if (!dims_ok(dims)) return -1;
  const int flags = (int)mode & ~0xff;
  if (flags & ~(int)SEER_SELECT_FORCE_DIAGONAL) return -1;
  const int fd = (flags & SEER_SELECT_FORCE_DIAGONAL) ? 1 : 0;
  const int nb = dims->n / seer::kBlock;
  switch ((int)mode & 0xff) {
    case SEER_SELECT_THRESHOLD: return nb;
    case SEER_SELECT_TOPK_K: return k < 1 ? -1 : (k + fd < nb ? k + fd : nb);
    case SEER_SELECT_TOPK_DENSITY: {
      if (!(density > 0.f && density <= 1.f)) return -1;
      int worst = 0;
      for (int i = 0; i < nb; ++i) {
        int ki = (int)std::ceil((double)(density * (float)(i + 1)));
        if (ki < 1) ki = 1;
        ki += fd;
        if (ki > i + 1) ki = i + 1;
        if (ki > worst) worst = ki;
      }
      return worst;
    }
  }
  return -1;
}

static seer_status check_select(const seer_dims* dims, seer_select_mode mode, float T, int32_t k,
                                float density, int32_t cap) {
  if ((int)mode & ~0xff & ~(int)SEER_SELECT_FORCE_DIAGONAL) return SEER_ERR_INVALID_ARG;
  switch ((int)mode & 0xff) {
    case SEER_SELECT_THRESHOLD:
      if (!(T > 0.f) || !std::isfinite(T)) return SEER_ERR_INVALID_ARG;
      break;
    case SEER_SELECT_TOPK_K:
      if (k < 1) return SEER_ERR_INVALID_ARG;
      break;
    case SEER_SELECT_TOPK_DENSITY:
      if (!(density > 0.f && density <= 1.f)) return SEER_ERR_INVALID_ARG;
      break;
    default:
      return SEER_ERR_INVALID_ARG;
  }
  if (cap < 1) return SEER_ERR_INVALID_ARG;
  if (cap < seer_gate_required_cap(dims, mode, k, density)) return SEER_ERR_CAPACITY;
  return SEER_OK;
}

namespace {
// The gate on a workspace laid out by gate_ws; `tab` is the varlen block
// table (null for the plain batched layout).
seer_status run_gate(const seer_dims* dims, const void* Q, const void* K, seer_dtype dtype, const float* Wq,
                     const float* Wk, int32_t h, float rope_theta, seer_select_mode mode, float T, int32_t k,
                     float density, float* scores_out, int32_t* counts, int32_t* indices, int32_t cap, void* ws,
                     const int2* tab, cudaStream_t st) {
  const GateWs w = gate_ws(dims, h);
  uint8_t* base = (uint8_t*)ws;
  float* qbar = (float*)(base + w.qbar);
  float* kbar = (float*)(base + w.kbar);
  float* qt = (float*)(base + w.qt);
  float* kt = (float*)(base + w.kt);
  float* logits = scores_out ? scores_out : (float*)(base + w.logits);
  const int B = dims->B, Hq = dims->Hq, Hkv = dims->Hkv, n = dims->n, d = dims->d;
  const int nb = n / seer::kBlock, G = Hq / Hkv;

  // q~ = Wq[hq] qbar, k~ = Wk[g] kbar (batch z = b*H + head; weights by head)
  const bool proj_tc = gate_proj_tf32x3(h, d);
  // without RoPE the projections write q~ and k~ already split for the logits
  const bool split_in_proj = proj_tc && gate_tf32x3(h) && !(rope_theta > 0.f);
  if (proj_tc) {
    // on the tensor cores, three tf32 products as for the logits; the pooling
    // writes qbar and kbar already split into their tf32 parts and remainders
    float* qbhi = (float*)(base + w.qbar_hi);
    float* qblo = (float*)(base + w.qbar_lo);
    float* kbhi = (float*)(base + w.kbar_hi);
    float* kblo = (float*)(base + w.kbar_lo);
    float* wqh = (float*)(base + w.wq_hi);
    float* wql = (float*)(base + w.wq_lo);
    float* wkh = (float*)(base + w.wk_hi);
    float* wkl = (float*)(base + w.wk_lo);
    seer::GateInputs gi;
    gi.Q = Q;
    gi.K = K;
    gi.nq = (long long)B * Hq * nb;
    gi.nk = (long long)B * Hkv * nb;
    gi.cq = (gi.nq + 7) / 8;
    gi.ck = (gi.nk + 7) / 8;
    gi.n = n;
    gi.d = d;
    gi.qhi = qbhi;
    gi.qlo = qblo;
    gi.khi = kbhi;
    gi.klo = kblo;
    gi.tab = tab;
    gi.Wq = Wq;
    gi.Wk = Wk;
    gi.nwq = (long long)Hq * h * d;
    gi.nwk = (long long)Hkv * h * 3 * d;
    gi.wqh = wqh;
    gi.wql = wql;
    gi.wkh = wkh;
    gi.wkl = wkl;
    SEER_CUDA(seer::launch_gate_inputs(gi, dtype, st));
    CUtensorMap tmAh, tmAl, tmBh, tmBl;
    seer::Tf32x3Params tp;
    tp.M = nb;
    tp.N = h;
    tp.ldc = h;
    tp.zmul = 0;
    tp.zg = 1;
    tp.causal = 0;
    tp.c_bs = (long long)nb * h;
    tp.alpha = 1.0f;
    tp.C_lo = nullptr;
    tp.tma_out = 1;
    tp.status = &((seer::WsHeader*)ws)->status;
    tp.timeout_ns = kTimeoutNs;
    if (!make_tmap_f32(&tmAh, qbhi, (long long)B * Hq * nb, d, 128) ||
        !make_tmap_f32(&tmAl, qblo, (long long)B * Hq * nb, d, 128) ||
        !make_tmap_f32(&tmBh, wqh, (long long)Hq * h, d, 128) || !make_tmap_f32(&tmBl, wql, (long long)Hq * h, d, 128))
      return cuda_fail(cudaErrorInvalidValue);
    tp.K = d;
    tp.zh = Hq;
    tp.C = qt;
    tp.C_lo = split_in_proj ? (float*)(base + w.qlo) : nullptr;
    CUtensorMap tmC, tmClo;
    if (!make_tmap_f32_batched(&tmC, qt, h, nb, B * Hq, h, (long long)nb * h) ||
        !make_tmap_f32_batched(&tmClo, tp.C_lo ? tp.C_lo : qt, h, nb, B * Hq, h, (long long)nb * h))
      return cuda_fail(cudaErrorInvalidValue);
    SEER_CUDA(seer::launch_gemm_tf32x3_causal(tmAh, tmAl, tmBh, tmBl, tmC, tmClo, tp, B * Hq, st));
    if (!make_tmap_f32(&tmAh, kbhi, (long long)B * Hkv * nb, 3 * d, 128) ||
        !make_tmap_f32(&tmAl, kblo, (long long)B * Hkv * nb, 3 * d, 128) ||
        !make_tmap_f32(&tmBh, wkh, (long long)Hkv * h, 3 * d, 128) ||
        !make_tmap_f32(&tmBl, wkl, (long long)Hkv * h, 3 * d, 128))
      return cuda_fail(cudaErrorInvalidValue);
    tp.K = 3 * d;
    tp.zh = Hkv;
    tp.C = kt;
    tp.C_lo = split_in_proj ? (float*)(base + w.klo) : nullptr;
    if (!make_tmap_f32_batched(&tmC, kt, h, nb, B * Hkv, h, (long long)nb * h) ||
        !make_tmap_f32_batched(&tmClo, tp.C_lo ? tp.C_lo : kt, h, nb, B * Hkv, h, (long long)nb * h))
      return cuda_fail(cudaErrorInvalidValue);
    SEER_CUDA(seer::launch_gemm_tf32x3_causal(tmAh, tmAl, tmBh, tmBl, tmC, tmClo, tp, B * Hkv, st));
  } else {
    SEER_CUDA(seer::launch_pool(Q, dtype, false, (long long)B * Hq, n, d, qbar, st, tab));
    SEER_CUDA(seer::launch_pool(K, dtype, true, (long long)B * Hkv, n, d, kbar, st, tab));
    SEER_CUDA(seer::launch_gemm_nt(qbar, Wq, qt, nb, h, d, (long long)nb * d, (long long)h * d,
                                   (long long)nb * h, h, B * Hq, Hq, 0, 1, 1.0f, false, st));
    SEER_CUDA(seer::launch_gemm_nt(kbar, Wk, kt, nb, h, 3 * d, (long long)nb * 3 * d,
                                   (long long)h * 3 * d, (long long)nb * h, h, B * Hkv, Hkv, 0, 1,
                                   1.0f, false, st));
  }
  if (rope_theta > 0.f) {
    SEER_CUDA(seer::launch_rope(qt, (long long)B * Hq * nb, nb, h, rope_theta, st));
    SEER_CUDA(seer::launch_rope(kt, (long long)B * Hkv * nb, nb, h, rope_theta, st));
  }
  // causal block logits q~_i . k~_j / sqrt(d), KV head of query head z%Hq
  const float alpha = (float)(1.0 / std::sqrt((double)d));
  if (gate_tf32x3(h)) {
    float* qlo = (float*)(base + w.qlo);
    float* klo = (float*)(base + w.klo);
    if (!split_in_proj) {
      SEER_CUDA(seer::launch_split_tf32(qt, qlo, (long long)B * Hq * nb * h, st));
      SEER_CUDA(seer::launch_split_tf32(kt, klo, (long long)B * Hkv * nb * h, st));
    }
    CUtensorMap tmAh, tmAl, tmBh, tmBl;
    if (!make_tmap_f32(&tmAh, qt, (long long)B * Hq * nb, h, 128) ||
        !make_tmap_f32(&tmAl, qlo, (long long)B * Hq * nb, h, 128) ||
        !make_tmap_f32(&tmBh, kt, (long long)B * Hkv * nb, h, 128) ||
        !make_tmap_f32(&tmBl, klo, (long long)B * Hkv * nb, h, 128))
      return cuda_fail(cudaErrorInvalidValue);
    seer::Tf32x3Params tp;
    tp.M = nb;
    tp.N = nb;
    tp.K = h;
    tp.ldc = nb;
    tp.zh = Hq;
    tp.zmul = Hkv;
    tp.zg = G;
    tp.causal = 1;
    tp.c_bs = (long long)nb * nb;
    tp.alpha = alpha;
    tp.C = logits;
    tp.C_lo = nullptr;
    tp.tma_out = 0;
    tp.status = &((seer::WsHeader*)ws)->status;
    tp.timeout_ns = kTimeoutNs;
    // each q~ row block held on chip while its key tiles stream past (h <= 128)
    if (seer::gemm_tf32x3_rows_fits(h, nb, tp.c_bs, logits)) {
      CUtensorMap tmAph, tmApl, tmC;
      if (!make_tmap_f32_panels(&tmAph, qt, (long long)B * Hq * nb, h, 128) ||
          !make_tmap_f32_panels(&tmApl, qlo, (long long)B * Hq * nb, h, 128) ||
          !make_tmap_f32_batched(&tmC, logits, nb, nb, B * Hq, nb, tp.c_bs))
        return cuda_fail(cudaErrorInvalidValue);
      SEER_CUDA(seer::launch_gemm_tf32x3_rows(tmAph, tmApl, tmBh, tmBl, tmC, tp, B * Hq, num_sms(), st));
    } else {
      SEER_CUDA(seer::launch_gemm_tf32x3_causal(tmAh, tmAl, tmBh, tmBl, tmAh, tmAh, tp, B * Hq, st));
    }
  } else {
    SEER_CUDA(seer::launch_gemm_nt(qt, kt, logits, nb, nb, h, (long long)nb * h, (long long)nb * h,
                                   (long long)nb * nb, nb, B * Hq, Hq, Hkv, G, alpha, true, st));
  }
  SEER_CUDA(seer::launch_row_select(logits, scores_out, true, (long long)B * Hq * nb, nb, (int)mode,
                                    T, k, density, counts, indices, cap, st, 0, tab));
  return SEER_OK;
}

seer_status check_gate_args(const seer_dims* dims, const void* Q, const void* K, seer_dtype dtype, const float* Wq,
                            const float* Wk, int32_t h, float rope_theta, seer_select_mode mode, float T, int32_t k,
                            float density, int32_t* counts, int32_t* indices, int32_t cap) {
  if (!dims_ok(dims) || !Q || !K || !Wq || !Wk || !counts || !indices) return SEER_ERR_INVALID_ARG;
  if (dtype != SEER_BF16 && dtype != SEER_FP32) return SEER_ERR_INVALID_ARG;
  if (h < 1 || h > 256 || (h % 4) != 0) return SEER_ERR_INVALID_ARG;
  if (!std::isfinite(rope_theta)) return SEER_ERR_INVALID_ARG;
  seer_status s = dims_supported(dims);
  if (s != SEER_OK) return s;
  if (!aligned(Q, 16) || !aligned(K, 16)) return SEER_ERR_INVALID_ARG;
  return check_select(dims, mode, T, k, density, cap);
}
}  // namespace

seer_status seer_gate(const seer_dims* dims, const void* Q, const void* K, seer_dtype dtype,
                      const float* Wq, const float* Wk, int32_t h, float rope_theta,
                      seer_select_mode mode, float T, int32_t k, float density, float* scores_out,
                      int32_t* counts, int32_t* indices, int32_t cap, void* ws, size_t ws_bytes,
                      seer_stream_t stream) {
  seer_status s = check_gate_args(dims, Q, K, dtype, Wq, Wk, h, rope_theta, mode, T, k, density, counts, indices, cap);
  if (s != SEER_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  s = begin_ws(ws, ws_bytes, gate_ws(dims, h).total, st);
  if (s != SEER_OK) return s;
  return run_gate(dims, Q, K, dtype, Wq, Wk, h, rope_theta, mode, T, k, density, scores_out, counts, indices, cap,
                  ws, nullptr, st);
}

size_t seer_gate_varlen_workspace_size(const seer_dims* dims, int32_t h) {
  if (!dims_ok(dims) || h < 1) return 0;
  seer::WsCarver c;
  c.off = gate_ws(dims, h).total;
  c.take(sizeof(int2) * (size_t)(dims->n / seer::kBlock));
  return c.off;
}

seer_status seer_gate_varlen(const seer_dims* dims, const void* Q, const void* K, seer_dtype dtype,
                             const float* Wq, const float* Wk, int32_t h, float rope_theta,
                             const int32_t* seq_start, const int32_t* seq_len, int32_t nseq,
                             seer_select_mode mode, float T, int32_t k, float density, float* scores_out,
                             int32_t* counts, int32_t* indices, int32_t cap, void* ws, size_t ws_bytes,
                             seer_stream_t stream) {
  seer_status s = check_gate_args(dims, Q, K, dtype, Wq, Wk, h, rope_theta, mode, T, k, density, counts, indices, cap);
  if (s != SEER_OK) return s;
  if (dims->B != 1 || !seq_start || !seq_len || nseq < 1) return SEER_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  s = begin_ws(ws, ws_bytes, seer_gate_varlen_workspace_size(dims, h), st);
  if (s != SEER_OK) return s;
  int2* tab = (int2*)((uint8_t*)ws + gate_ws(dims, h).total);
  SEER_CUDA(seer::launch_varlen_table(seq_start, seq_len, nseq, dims->n, tab, &((seer::WsHeader*)ws)->status, st));
  return run_gate(dims, Q, K, dtype, Wq, Wk, h, rope_theta, mode, T, k, density, scores_out, counts, indices, cap,
                  ws, tab, st);
}

seer_status seer_gate_select(const seer_dims* dims, const float* scores, seer_select_mode mode,
                             float T, int32_t k, float density, int32_t* counts, int32_t* indices,
                             int32_t cap, seer_stream_t stream) {
  if (!dims_ok(dims) || !scores || !counts || !indices) return SEER_ERR_INVALID_ARG;
  if (dims->block != seer::kBlock) return SEER_ERR_UNSUPPORTED;
  seer_status s = check_select(dims, mode, T, k, density, cap);
  if (s != SEER_OK) return s;
  const int nb = dims->n / seer::kBlock;
  SEER_CUDA(seer::launch_row_select(scores, nullptr, false, (long long)dims->B * dims->Hq * nb, nb,
                                    (int)mode, T, k, density, counts, indices, cap,
                                    (cudaStream_t)stream));
  return SEER_OK;
}

// ---------------------------------------------------------- sparse attn ---
size_t seer_sparse_attn_workspace_size(const seer_dims* dims, seer_dtype dtype) {
  if (!dims_ok(dims)) return 0;
  return attn_ws(dims, dtype).total;
}

seer_status seer_sparse_attn(const seer_dims* dims, const void* Q, const void* K, const void* V,
                             seer_dtype dtype, const int32_t* counts, const int32_t* indices,
                             int32_t cap, float scale, void* O, float* lse, void* ws,
                             size_t ws_bytes, seer_stream_t stream) {
  if (!dims_ok(dims) || !Q || !K || !V || !O || !counts || !indices) return SEER_ERR_INVALID_ARG;
  if (dtype != SEER_BF16 && dtype != SEER_FP32) return SEER_ERR_INVALID_ARG;
  if (cap < 1 || !(scale >= 0.f) || !std::isfinite(scale)) return SEER_ERR_INVALID_ARG;
  seer_status s = dims_supported(dims);
  if (s != SEER_OK) return s;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16))
    return SEER_ERR_INVALID_ARG;
  const AttnWs w = attn_ws(dims, dtype);
  cudaStream_t st = (cudaStream_t)stream;
  s = begin_ws(ws, ws_bytes, w.total, st);
  if (s != SEER_OK) return s;
  uint8_t* base = (uint8_t*)ws;
  const int B = dims->B, Hq = dims->Hq, Hkv = dims->Hkv, n = dims->n, d = dims->d;
  const void *q = Q, *v16 = V;
  if (dtype == SEER_FP32) {
    SEER_CUDA(to_bf16(Q, base + w.q16, (long long)B * Hq * n * d, st));
    SEER_CUDA(to_bf16(V, base + w.v16, (long long)B * Hkv * n * d, st));
    q = base + w.q16;
    v16 = base + w.v16;
  }
  seer::WsHeader* hdr = (seer::WsHeader*)ws;
  // bf16 inputs: a device-side check picks the 128-row dense kernel when the
  // lists are the all-ones causal mask (every count is i + 1); the sparse
  // kernels then return at once, and the other way round
  const bool dual = dtype == SEER_BF16;
  uint32_t* not_dense = &hdr->pad[kWsNotDenseWord];
  if (dual) SEER_CUDA(seer::launch_dense_check(counts, (long long)B * Hq * (n / seer::kBlock), n / seer::kBlock, not_dense, st));
  const long long records = (long long)B * Hkv * (n / seer::kBlock);
  SEER_CUDA(seer::launch_kt_tiles(K, dtype == SEER_FP32, base + w.kt, records, n, d, st, dual ? not_dense : nullptr));
  CUtensorMap tmQ, tmKt, tmV;
  if (!make_tmap_bf16_panels(&tmQ, q, (long long)B * Hq * n, d, 64) ||
      !make_tmap_rows(&tmKt, base + w.kt, records * d, d) ||
      !make_tmap_bf16_panels(&tmV, v16, (long long)B * Hkv * n, d, 64))
    return cuda_fail(cudaErrorInvalidValue);
  seer::AttnParams p{};
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.n = n;
  p.d = d;
  p.nb = n / seer::kBlock;
  p.G = Hq / Hkv;
  p.cap = cap;
  p.total_units = (long long)B * Hq * p.nb;
  p.counts = counts;
  p.indices = indices;
  p.dense = 0;
  p.O = O;
  p.lse = lse;
  p.out_fp32 = dtype == SEER_FP32;
  const double sc = scale > 0.f ? (double)scale : 1.0 / std::sqrt((double)d);
  p.scale_log2 = (float)(sc * 1.4426950408889634);
  p.status = &hdr->status;
  p.work_counter = &hdr->work_counter;
  p.timeout_ns = kTimeoutNs;
  p.trace = reinterpret_cast<unsigned long long*>(hdr->pad + 4);  // 16 x u64 in the header
  p.redo_count = &hdr->work_counter2;
  p.redo_list = reinterpret_cast<int*>(base + w.redo);
  p.redo_cap = (int)p.total_units;
  p.map = nullptr;
  p.test_skip_qk_commit = g_test_skip_qk_commit;
  p.k_rows = 0;
  if (g_test_wait_limit_ns) p.timeout_ns = g_test_wait_limit_ns;
  p.run_if = dual ? not_dense : nullptr;
  p.run_if_value = 1;
  SEER_CUDA(seer::launch_empty_rows(p, st));
  SEER_CUDA(seer::launch_sparse_attn(tmQ, tmKt, tmV, p, num_sms(), st));
  SEER_CUDA(seer::launch_sparse_attn_redo(q, base + w.kt, v16, p, st));
  if (dual) {
    // the dense path: 128-row query tiles over every causal key block, P in
    // TMEM (the training forward's kernel without the map)
    CUtensorMap tmQ2, tmK2, tmV2;
    if (!make_tmap_bf16_panels(&tmQ2, q, (long long)B * Hq * n, d, 128) ||
        !make_tmap_bf16_panels(&tmK2, K, (long long)B * Hkv * n, d, 128) ||
        !make_tmap_bf16_panels(&tmV2, v16, (long long)B * Hkv * n, d, 128))
      return cuda_fail(cudaErrorInvalidValue);
    seer::FwdParams f{};
    f.B = B;
    f.Hq = Hq;
    f.Hkv = Hkv;
    f.n = n;
    f.d = d;
    f.nb = p.nb;
    f.G = p.G;
    f.npairs = (p.nb + 1) / 2;
    f.total_units = (long long)B * Hq * f.npairs;
    f.O = O;
    f.out_fp32 = 0;
    f.lse = lse;
    f.map = nullptr;
    f.scale_log2 = p.scale_log2;
    f.r = nullptr;
    f.status = p.status;
    f.work_counter = p.work_counter;
    f.timeout_ns = p.timeout_ns;
    f.redo_count = p.redo_count;
    f.redo_list = p.redo_list;
    f.redo_cap = p.redo_cap;
    f.run_if = not_dense;
    f.run_if_value = 0;
    SEER_CUDA(seer::launch_fwd(tmQ2, tmK2, tmV2, f, num_sms(), st));
    // its exact fallback reads K as rows
    seer::AttnParams a = p;
    a.dense = 1;
    a.k_rows = 1;
    a.run_if_value = 0;
    SEER_CUDA(seer::launch_sparse_attn_redo(q, K, v16, a, st));
  }
  return SEER_OK;
}

// -------------------------------------------------------------- blockmax --
size_t seer_blockmax_workspace_size(const seer_dims* dims, seer_dtype dtype) {
  if (!dims_ok(dims)) return 0;
  return bmax_ws(dims, dtype, num_sms()).total;
}

seer_status seer_attn_blockmax(const seer_dims* dims, const void* Q, const void* K,
                               seer_dtype dtype, float scale, float* map_out, float* lse_out,
                               void* ws, size_t ws_bytes, seer_stream_t stream) {
  if (!dims_ok(dims) || !Q || !K || !map_out) return SEER_ERR_INVALID_ARG;
  if (dtype != SEER_BF16 && dtype != SEER_FP32) return SEER_ERR_INVALID_ARG;
  if (!(scale >= 0.f) || !std::isfinite(scale)) return SEER_ERR_INVALID_ARG;
  seer_status s = dims_supported(dims);
  if (s != SEER_OK) return s;
  if (!aligned(Q, 16) || !aligned(K, 16)) return SEER_ERR_INVALID_ARG;
  const int sms = num_sms();
  const BmaxWs w = bmax_ws(dims, dtype, sms);
  cudaStream_t st = (cudaStream_t)stream;
  s = begin_ws(ws, ws_bytes, w.total, st);
  if (s != SEER_OK) return s;
  uint8_t* base = (uint8_t*)ws;
  const int B = dims->B, Hq = dims->Hq, Hkv = dims->Hkv, n = dims->n, d = dims->d;
  const void *q = Q, *k = K;
  if (dtype == SEER_FP32) {
    SEER_CUDA(to_bf16(Q, base + w.q16, (long long)B * Hq * n * d, st));
    SEER_CUDA(to_bf16(K, base + w.k16, (long long)B * Hkv * n * d, st));
    q = base + w.q16;
    k = base + w.k16;
  }
  CUtensorMap tmQ, tmK;
  if (!make_tmap(&tmQ, q, (long long)B * Hq * n, d, 128) ||
      !make_tmap(&tmK, k, (long long)B * Hkv * n, d, 128))
    return cuda_fail(cudaErrorInvalidValue);
  seer::BmaxParams p;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.n = n;
  p.d = d;
  p.nb = n / seer::kBlock;
  p.G = Hq / Hkv;
  p.npairs = (p.nb + 1) / 2;
  p.total_units = (long long)B * Hq * p.npairs;
  p.map = map_out;
  p.lse = lse_out;
  const double sc = scale > 0.f ? (double)scale : 1.0 / std::sqrt((double)d);
  p.scale_log2 = (float)(sc * 1.4426950408889634);
  p.r = (float*)(base + w.r);
  seer::WsHeader* hdr = (seer::WsHeader*)ws;
  p.status = &hdr->status;
  p.work_counter = &hdr->work_counter;
  p.timeout_ns = kTimeoutNs;
  SEER_CUDA(seer::launch_blockmax(tmQ, tmK, p, w.ctas, st));
  return SEER_OK;
}

// ----------------------------------------------------------- tf32 attn ---
size_t seer_sparse_attn_tf32_workspace_size(const seer_dims* dims) {
  if (!dims_ok(dims)) return 0;
  seer::WsCarver c;  // V^T per key block
  c.take(sizeof(float) * (size_t)dims->B * dims->Hkv * dims->n * dims->d);
  return c.off;
}

seer_status seer_sparse_attn_tf32(const seer_dims* dims, const float* Q, const float* K, const float* V,
                                  const int32_t* counts, const int32_t* indices, int32_t cap, float scale, float* O,
                                  float* lse, void* ws, size_t ws_bytes, seer_stream_t stream) {
  if (!dims_ok(dims) || !Q || !K || !V || !O || !counts || !indices) return SEER_ERR_INVALID_ARG;
  if (cap < 1 || !(scale >= 0.f) || !std::isfinite(scale)) return SEER_ERR_INVALID_ARG;
  seer_status s = dims_supported(dims);
  if (s != SEER_OK) return s;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16)) return SEER_ERR_INVALID_ARG;
  if ((long long)dims->B * dims->Hq * (dims->n / seer::kBlock) >= (1LL << 31)) return SEER_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  s = begin_ws(ws, ws_bytes, seer_sparse_attn_tf32_workspace_size(dims), st);
  if (s != SEER_OK) return s;
  const int B = dims->B, Hq = dims->Hq, Hkv = dims->Hkv, n = dims->n, d = dims->d;
  float* Vt = (float*)((uint8_t*)ws + sizeof(seer::WsHeader));
  CUtensorMap tmQ, tmK, tmV;
  if (!make_tmap_f32_panels(&tmQ, Q, (long long)B * Hq * n, d, 64) ||
      !make_tmap_f32_panels(&tmK, K, (long long)B * Hkv * n, d, 64) ||
      !make_tmap_f32_panels(&tmV, Vt, (long long)B * Hkv * n * d / 64, 64, d))
    return cuda_fail(cudaErrorInvalidValue);
  SEER_CUDA(seer::launch_vt(V, Vt, (long long)B * Hkv, n, d, st));
  seer::Tf32AttnParams p{};
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.n = n;
  p.d = d;
  p.nb = n / seer::kBlock;
  p.cap = cap;
  p.total_units = (long long)B * Hq * p.nb;
  p.counts = counts;
  p.indices = indices;
  p.O = O;
  p.lse = lse;
  const double sc = scale > 0.f ? (double)scale : 1.0 / std::sqrt((double)d);
  p.scale_log2 = (float)(sc * 1.4426950408889634);
  p.status = &((seer::WsHeader*)ws)->status;
  p.timeout_ns = kTimeoutNs;
  SEER_CUDA(seer::launch_attn_tf32(tmQ, tmK, tmV, p, st));
  return SEER_OK;
}

// ---------------------------------------------------------- decode stage --
namespace {
// Largest list a decode row can need: c candidates, the prefill rules.
int decode_required_cap(seer_select_mode mode, int32_t k, float density, int c) {
  if (c <= 0) return 0;
  if (mode == SEER_SELECT_TOPK_K) return k < c ? k : c;
  if (mode == SEER_SELECT_TOPK_DENSITY) {
    int kk = (int)std::ceil((double)(density * (float)c));
    return kk < 1 ? 1 : (kk > c ? c : kk);
  }
  return c;
}
bool decode_len_ok(const seer_dims* d, int32_t seq_len) { return seq_len >= 1 && seq_len <= d->n; }

struct DecAttnWs {
  size_t ticket, part, total;
  int splits;
};
DecAttnWs dec_attn_ws(const seer_dims* d) {
  const long long rows = (long long)d->B * d->Hq;
  DecAttnWs w;
  w.splits = seer::decode_attn_splits(rows);
  seer::WsCarver c;
  w.ticket = c.take(sizeof(int32_t) * (size_t)rows);
  w.part = c.take(sizeof(float) * (size_t)rows * w.splits * (d->d + 2));
  w.total = c.off;
  return w;
}

struct DecGtWs {
  size_t ticket, stats, total;
};
DecGtWs dec_gt_ws(const seer_dims* d) {
  const long long rows = (long long)d->B * d->Hq;
  DecGtWs w;
  seer::WsCarver c;
  w.ticket = c.take(sizeof(int32_t) * (size_t)rows);
  w.stats = c.take(sizeof(float) * 2 * (size_t)rows * seer::kGtMaxChunks);
  w.total = c.off;
  return w;
}
}  // namespace

size_t seer_decode_gate_workspace_size(const seer_dims* dims) {
  if (!dims_ok(dims)) return 0;
  seer::WsCarver c;
  c.take(sizeof(float) * (size_t)dims->B * dims->Hq * (dims->n / seer::kBlock));
  return c.off;
}

size_t seer_sparse_decode_attn_workspace_size(const seer_dims* dims) {
  if (!dims_ok(dims)) return 0;
  return dec_attn_ws(dims).total;
}

size_t seer_decode_blockmax_workspace_size(const seer_dims* dims) {
  if (!dims_ok(dims)) return 0;
  return dec_gt_ws(dims).total;
}

seer_status seer_decode_kcache_update(const seer_dims* dims, const void* Kcache, seer_dtype dtype, const float* Wk,
                                      int32_t h, int32_t block_begin, int32_t block_end, float* kt_cache,
                                      seer_stream_t stream) {
  if (!dims_ok(dims) || !Kcache || !Wk || !kt_cache) return SEER_ERR_INVALID_ARG;
  if (dtype != SEER_BF16 && dtype != SEER_FP32) return SEER_ERR_INVALID_ARG;
  seer_status s = dims_supported(dims);
  if (s != SEER_OK) return s;
  if (h != dims->d) return SEER_ERR_INVALID_ARG;  // the token's q meets k~ directly
  if (!aligned(Kcache, 16) || !aligned(kt_cache, 16)) return SEER_ERR_INVALID_ARG;
  const int nb = dims->n / seer::kBlock;
  if (block_begin < 0 || block_end < block_begin || block_end > nb) return SEER_ERR_INVALID_ARG;
  if (block_end == block_begin) return SEER_OK;
  SEER_CUDA(seer::launch_kcache(Kcache, dtype == SEER_FP32, Wk, kt_cache, (long long)dims->B * dims->Hkv, dims->Hkv,
                                dims->n, dims->d, block_begin, block_end - block_begin, (cudaStream_t)stream));
  return SEER_OK;
}

int32_t seer_decode_gate_required_cap(const seer_dims* dims, int32_t seq_len, seer_select_mode mode, int32_t k,
                                      float density) {
  if (!dims_ok(dims) || !decode_len_ok(dims, seq_len)) return -1;
  if ((int)mode & ~0xff & ~(int)SEER_SELECT_FORCE_DIAGONAL) return -1;
  // the token's own block is always attended: the diagonal flag changes nothing
  mode = (seer_select_mode)((int)mode & 0xff);
  return decode_required_cap(mode, k, density, (seq_len - 1) / seer::kBlock);
}

seer_status seer_decode_gate(const seer_dims* dims, const void* q, seer_dtype dtype, const float* kt_cache,
                             int32_t seq_len, seer_select_mode mode, float T, int32_t k, float density,
                             float* scores_out, int32_t* counts, int32_t* indices, int32_t cap, void* ws,
                             size_t ws_bytes, seer_stream_t stream) {
  if (!dims_ok(dims) || !q || !kt_cache || !counts || !indices) return SEER_ERR_INVALID_ARG;
  if (dtype != SEER_BF16 && dtype != SEER_FP32) return SEER_ERR_INVALID_ARG;
  seer_status s = dims_supported(dims);
  if (s != SEER_OK) return s;
  if (!decode_len_ok(dims, seq_len) || !aligned(kt_cache, 16)) return SEER_ERR_INVALID_ARG;
  if ((int)mode & ~0xff & ~(int)SEER_SELECT_FORCE_DIAGONAL) return SEER_ERR_INVALID_ARG;
  // the token's own block is always attended: the diagonal flag changes nothing
  mode = (seer_select_mode)((int)mode & 0xff);
  if (mode == SEER_SELECT_THRESHOLD && !(T > 0.f)) return SEER_ERR_INVALID_ARG;
  if (mode == SEER_SELECT_TOPK_K && k < 1) return SEER_ERR_INVALID_ARG;
  if (mode == SEER_SELECT_TOPK_DENSITY && !(density > 0.f && density <= 1.f)) return SEER_ERR_INVALID_ARG;
  if (mode != SEER_SELECT_THRESHOLD && mode != SEER_SELECT_TOPK_K && mode != SEER_SELECT_TOPK_DENSITY)
    return SEER_ERR_INVALID_ARG;
  const int c = (seq_len - 1) / seer::kBlock;
  if (cap < decode_required_cap(mode, k, density, c) || cap < 1) return SEER_ERR_CAPACITY;
  cudaStream_t st = (cudaStream_t)stream;
  s = begin_ws(ws, ws_bytes, seer_decode_gate_workspace_size(dims), st);
  if (s != SEER_OK) return s;
  const long long rows = (long long)dims->B * dims->Hq;
  if (c == 0) {  // no complete block yet: nothing to select
    SEER_CUDA(cudaMemsetAsync(counts, 0, sizeof(int32_t) * rows, st));
    return SEER_OK;
  }
  float* logits = (float*)((uint8_t*)ws + sizeof(seer::WsHeader));
  SEER_CUDA(seer::launch_decode_logits(q, dtype == SEER_FP32, kt_cache, logits, dims->B, dims->Hq, dims->Hkv,
                                       dims->d, c, dims->n / seer::kBlock, (float)(1.0 / std::sqrt((double)dims->d)),
                                       st));
  SEER_CUDA(seer::launch_row_select(logits, scores_out, true, rows, c, (int)mode, T, k, density, counts, indices, cap,
                                    st, c));
  return SEER_OK;
}

seer_status seer_sparse_decode_attn(const seer_dims* dims, const void* q, const void* Kcache, const void* Vcache,
                                    seer_dtype dtype, int32_t seq_len, const int32_t* counts, const int32_t* indices,
                                    int32_t cap, float scale, void* O, float* lse, void* ws, size_t ws_bytes,
                                    seer_stream_t stream) {
  if (!dims_ok(dims) || !q || !Kcache || !Vcache || !counts || !indices || !O) return SEER_ERR_INVALID_ARG;
  if (dtype != SEER_BF16 && dtype != SEER_FP32) return SEER_ERR_INVALID_ARG;
  if (cap < 1 || !(scale >= 0.f) || !std::isfinite(scale)) return SEER_ERR_INVALID_ARG;
  seer_status s = dims_supported(dims);
  if (s != SEER_OK) return s;
  if (!decode_len_ok(dims, seq_len)) return SEER_ERR_INVALID_ARG;
  if (!aligned(Kcache, 16) || !aligned(Vcache, 16)) return SEER_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const DecAttnWs w = dec_attn_ws(dims);
  s = begin_ws(ws, ws_bytes, w.total, st);
  if (s != SEER_OK) return s;
  const long long rows = (long long)dims->B * dims->Hq;
  SEER_CUDA(cudaMemsetAsync((uint8_t*)ws + w.ticket, 0, sizeof(int32_t) * rows, st));
  seer::DecodeAttnArgs a{};
  a.q = q;
  a.K = Kcache;
  a.V = Vcache;
  a.fp32 = dtype == SEER_FP32;
  a.counts = counts;
  a.indices = indices;
  a.cap = cap;
  a.Hq = dims->Hq;
  a.Hkv = dims->Hkv;
  a.d = dims->d;
  a.n_cap = dims->n;
  a.seq_len = seq_len;
  a.rows = rows;
  a.splits = w.splits;
  const double sc = scale > 0.f ? (double)scale : 1.0 / std::sqrt((double)dims->d);
  a.scale_log2 = (float)(sc * 1.4426950408889634);
  a.part = (float*)((uint8_t*)ws + w.part);
  a.ticket = (int32_t*)((uint8_t*)ws + w.ticket);
  a.O = O;
  a.lse = lse;
  a.status = &((seer::WsHeader*)ws)->status;
  a.timeout_ns = kTimeoutNs;
  SEER_CUDA(seer::launch_decode_attn(a, st));
  return SEER_OK;
}

seer_status seer_decode_blockmax(const seer_dims* dims, const void* q, const void* Kcache, seer_dtype dtype,
                                 int32_t seq_len, float scale, float* gt_out, float* lse_out, void* ws,
                                 size_t ws_bytes, seer_stream_t stream) {
  if (!dims_ok(dims) || !q || !Kcache || !gt_out) return SEER_ERR_INVALID_ARG;
  if (dtype != SEER_BF16 && dtype != SEER_FP32) return SEER_ERR_INVALID_ARG;
  if (!(scale >= 0.f) || !std::isfinite(scale)) return SEER_ERR_INVALID_ARG;
  seer_status s = dims_supported(dims);
  if (s != SEER_OK) return s;
  if (!decode_len_ok(dims, seq_len) || !aligned(Kcache, 16)) return SEER_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const DecGtWs w = dec_gt_ws(dims);
  s = begin_ws(ws, ws_bytes, w.total, st);
  if (s != SEER_OK) return s;
  SEER_CUDA(cudaMemsetAsync((uint8_t*)ws + w.ticket, 0, sizeof(int32_t) * (size_t)dims->B * dims->Hq, st));
  const double sc = scale > 0.f ? (double)scale : 1.0 / std::sqrt((double)dims->d);
  SEER_CUDA(seer::launch_decode_gt(q, Kcache, dtype == SEER_FP32, dims->B, dims->Hq, dims->Hkv, dims->d, dims->n,
                                   seq_len, (float)(sc * 1.4426950408889634), gt_out, lse_out,
                                   (float*)((uint8_t*)ws + w.stats), (int32_t*)((uint8_t*)ws + w.ticket),
                                   &((seer::WsHeader*)ws)->status, kTimeoutNs, st));
  return SEER_OK;
}

// --------------------------------------------------- training forward ----
namespace {
// The training forward's workspace: bf16 copies of fp32 inputs, the exact
// fallback's unit list, then the map scratch of every CTA ([nb][2][128] fp32).
struct FwdWs {
  size_t q16, k16, v16, redo, r, total;
  int ctas;
};

FwdWs fwd_ws(const seer_dims* d, seer_dtype dt, int sms) {
  seer::WsCarver c;
  FwdWs w{0, 0, 0, 0, 0, 0, sms};
  if (dt == SEER_FP32) {
    w.q16 = c.take(2ull * d->B * d->Hq * d->n * d->d);
    w.k16 = c.take(2ull * d->B * d->Hkv * d->n * d->d);
    w.v16 = c.take(2ull * d->B * d->Hkv * d->n * d->d);
  }
  w.redo = c.take(sizeof(int32_t) * (size_t)d->B * d->Hq * (d->n / seer::kBlock));
  w.r = c.take(sizeof(float) * (size_t)sms * (d->n / seer::kBlock) * 256);
  w.total = c.off;
  return w;
}
}  // namespace

size_t seer_attn_forward_map_workspace_size(const seer_dims* dims, seer_dtype dtype) {
  if (!dims_ok(dims)) return 0;
  return fwd_ws(dims, dtype, num_sms()).total;
}

seer_status seer_attn_forward_map(const seer_dims* dims, const void* Q, const void* K, const void* V,
                                  seer_dtype dtype, float scale, void* O, float* lse, float* map_out, void* ws,
                                  size_t ws_bytes, seer_stream_t stream) {
  if (!dims_ok(dims) || !Q || !K || !V || !O || !map_out) return SEER_ERR_INVALID_ARG;
  if (dtype != SEER_BF16 && dtype != SEER_FP32) return SEER_ERR_INVALID_ARG;
  if (!(scale >= 0.f) || !std::isfinite(scale)) return SEER_ERR_INVALID_ARG;
  seer_status s = dims_supported(dims);
  if (s != SEER_OK) return s;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16)) return SEER_ERR_INVALID_ARG;
  const int sms = num_sms();
  const FwdWs w = fwd_ws(dims, dtype, sms);
  cudaStream_t st = (cudaStream_t)stream;
  s = begin_ws(ws, ws_bytes, w.total, st);
  if (s != SEER_OK) return s;
  uint8_t* base = (uint8_t*)ws;
  const int B = dims->B, Hq = dims->Hq, Hkv = dims->Hkv, n = dims->n, d = dims->d;
  const void *q = Q, *k = K, *v = V;
  if (dtype == SEER_FP32) {
    SEER_CUDA(to_bf16(Q, base + w.q16, (long long)B * Hq * n * d, st));
    SEER_CUDA(to_bf16(K, base + w.k16, (long long)B * Hkv * n * d, st));
    SEER_CUDA(to_bf16(V, base + w.v16, (long long)B * Hkv * n * d, st));
    q = base + w.q16;
    k = base + w.k16;
    v = base + w.v16;
  }
  // one pass over 128-row query tiles: O, LSE and the map (the map's entries
  // above the diagonal stay 0)
  CUtensorMap tmQ, tmK, tmV;
  if (!make_tmap_bf16_panels(&tmQ, q, (long long)B * Hq * n, d, 128) ||
      !make_tmap_bf16_panels(&tmK, k, (long long)B * Hkv * n, d, 128) ||
      !make_tmap_bf16_panels(&tmV, v, (long long)B * Hkv * n, d, 128))
    return cuda_fail(cudaErrorInvalidValue);
  seer::WsHeader* hdr = (seer::WsHeader*)ws;
  seer::FwdParams p{};
  p.run_if = nullptr;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.n = n;
  p.d = d;
  p.nb = n / seer::kBlock;
  p.G = Hq / Hkv;
  p.npairs = (p.nb + 1) / 2;
  p.total_units = (long long)B * Hq * p.npairs;
  p.O = O;
  p.out_fp32 = dtype == SEER_FP32;
  p.lse = lse;
  p.map = map_out;
  const double sc = scale > 0.f ? (double)scale : 1.0 / std::sqrt((double)d);
  p.scale_log2 = (float)(sc * 1.4426950408889634);
  p.r = (float*)(base + w.r);
  p.status = &hdr->status;
  p.work_counter = &hdr->work_counter;
  p.timeout_ns = kTimeoutNs;
  p.redo_count = &hdr->work_counter2;
  p.redo_list = reinterpret_cast<int*>(base + w.redo);
  p.redo_cap = (int)((long long)B * Hq * p.nb);
  SEER_CUDA(cudaMemsetAsync(map_out, 0, sizeof(float) * (size_t)B * Hq * p.nb * p.nb, st));
  SEER_CUDA(seer::launch_fwd(tmQ, tmK, tmV, p, w.ctas, st));
  // the exact fallback for units whose scores rose far above their first
  // step's maximum (returns at once when there are none)
  seer::AttnParams a{};
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.n = n;
  a.d = d;
  a.nb = p.nb;
  a.G = p.G;
  a.cap = p.nb;
  a.total_units = (long long)B * Hq * p.nb;
  a.dense = 1;
  a.O = O;
  a.lse = lse;
  a.out_fp32 = p.out_fp32;
  a.scale_log2 = p.scale_log2;
  a.status = p.status;
  a.timeout_ns = kTimeoutNs;
  a.redo_count = p.redo_count;
  a.redo_list = p.redo_list;
  a.redo_cap = p.redo_cap;
  a.map = map_out;
  a.test_skip_qk_commit = -1;
  a.k_rows = 1;
  SEER_CUDA(seer::launch_sparse_attn_redo(q, k, v, a, st));
  return SEER_OK;
}

// ------------------------------------------------ prefill from host memory --
// The layer is processed in chunks of query heads that share a KV head: each
// KV head's K and V are copied in once (with its first chunk), each chunk's Q
// in on a copy stream, its gate and attention run on the caller's stream,
// its O (and LSE) go out on a third stream.  Two slots for chunks and two
// for KV heads let the copies of one chunk overlap the compute of its
// neighbours; small chunks keep the unoverlapped start (first copy in) and
// end (last compute and copy out) short.
namespace {
constexpr int kHostSlots = 2;

struct HostPlan {
  seer_dims g;  // one chunk: B = 1, Hq = C query heads, Hkv = 1
  int G = 0, C = 0, cap = 0, chunks = 0, per_kv = 0;
  size_t q = 0, kv = 0, o = 0, lse = 0, cnt = 0, idx = 0;                        // bytes
  size_t s_q = 0, s_o = 0, s_lse = 0, s_cnt = 0, s_idx = 0, slot = 0;            // chunk slot layout
  size_t s_k = 0, s_v = 0, kvslot = 0, kv_base = 0;                              // KV-head slot layout
  size_t gate_ws = 0, gate_ws_bytes = 0, attn_ws = 0, attn_ws_bytes = 0, status = 0, total = 0;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool host_plan(const seer_dims* dims, seer_dtype dtype, int32_t h, seer_select_mode mode, int32_t k, float density,
               HostPlan* P) {
  if (!dims_ok(dims) || (dtype != SEER_BF16 && dtype != SEER_FP32) || h < 1) return false;
  HostPlan p;
  p.G = dims->Hq / dims->Hkv;
  p.C = p.G % 2 == 0 ? p.G / 2 : p.G;  // two chunks per KV head when the group splits evenly
  p.per_kv = p.G / p.C;
  p.chunks = dims->B * dims->Hkv * p.per_kv;
  p.g = *dims;
  p.g.B = 1;
  p.g.Hq = p.C;
  p.g.Hkv = 1;
  p.cap = seer_gate_required_cap(&p.g, mode, k, density);
  if (p.cap < 1) return false;
  const size_t es = dtype == SEER_FP32 ? 4 : 2;
  const size_t n = (size_t)dims->n, d = (size_t)dims->d, nb = n / seer::kBlock;
  p.q = (size_t)p.C * n * d * es;
  p.kv = n * d * es;
  p.o = p.q;
  p.lse = (size_t)p.C * n * sizeof(float);
  p.cnt = (size_t)p.C * nb * sizeof(int32_t);
  p.idx = (size_t)p.C * nb * p.cap * sizeof(int32_t);
  size_t off = 0;
  p.s_q = off;
  off += align256(p.q);
  p.s_o = off;
  off += align256(p.o);
  p.s_lse = off;
  off += align256(p.lse);
  p.s_cnt = off;
  off += align256(p.cnt);
  p.s_idx = off;
  off += align256(p.idx);
  p.slot = off;
  p.kv_base = kHostSlots * p.slot;
  p.s_k = 0;
  p.s_v = align256(p.kv);
  p.kvslot = 2 * align256(p.kv);
  off = p.kv_base + kHostSlots * p.kvslot;
  p.gate_ws_bytes = seer_gate_workspace_size(&p.g, h);
  p.attn_ws_bytes = seer_sparse_attn_workspace_size(&p.g, dtype);
  if (p.gate_ws_bytes == 0 || p.attn_ws_bytes == 0) return false;
  p.gate_ws = off;
  off += align256(p.gate_ws_bytes);
  p.attn_ws = off;
  off += align256(p.attn_ws_bytes);
  p.status = off;  // two device status words per chunk (gate, attention)
  off += align256(sizeof(uint32_t) * 2 * (size_t)p.chunks);
  p.total = off;
  *P = p;
  return true;
}

// The streams and events of the host-memory pipeline, made once per device
// and host thread on first use (a call synchronises before it returns, so
// the calls of one thread never share them concurrently) and released when
// the thread exits.
struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr;
  cudaEvent_t copied_in[kHostSlots] = {}, computed[kHostSlots] = {}, copied_out[kHostSlots] = {};
  cudaEvent_t kv_in[kHostSlots] = {}, kv_done[kHostSlots] = {};
  ~HostPipe() {
    if (in) cudaStreamDestroy(in);
    if (out) cudaStreamDestroy(out);
    if (start) cudaEventDestroy(start);
    for (int s = 0; s < kHostSlots; ++s)
      for (cudaEvent_t e : {copied_in[s], computed[s], copied_out[s], kv_in[s], kv_done[s]})
        if (e) cudaEventDestroy(e);
  }
  cudaError_t create() {
    cudaError_t e = cudaStreamCreateWithFlags(&in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&out, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&start, cudaEventDisableTiming);
    for (int s = 0; s < kHostSlots && e == cudaSuccess; ++s)
      for (cudaEvent_t* ev : {&copied_in[s], &computed[s], &copied_out[s], &kv_in[s], &kv_done[s]})
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    return e;
  }
};

constexpr int kMaxPipeDevices = 64;

// This host thread's pipeline on the current device, or null (with *err set).
HostPipe* host_pipe(cudaError_t* err) {
  thread_local HostPipe pipes[kMaxPipeDevices];
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxPipeDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  HostPipe& p = pipes[dev];
  if (!p.in) {
    *err = p.create();
    if (*err != cudaSuccess) {
      p.~HostPipe();
      new (&p) HostPipe();
      return nullptr;
    }
  }
  return &p;
}
}  // namespace

size_t seer_prefill_host_buffer_size(const seer_dims* dims, seer_dtype dtype, int32_t h, seer_select_mode mode,
                                     int32_t k, float density) {
  HostPlan p;
  return host_plan(dims, dtype, h, mode, k, density, &p) ? p.total : 0;
}

seer_status seer_prefill_host(const seer_dims* dims, const void* hQ, const void* hK, const void* hV,
                              seer_dtype dtype, const float* Wq, const float* Wk, int32_t h, float rope_theta,
                              seer_select_mode mode, float T, int32_t k, float density, float scale, void* hO,
                              float* hLSE, void* dbuf, size_t dbuf_bytes, seer_stream_t stream) {
  if (!hQ || !hK || !hV || !hO || !Wq || !Wk) return SEER_ERR_INVALID_ARG;
  HostPlan P;
  if (!host_plan(dims, dtype, h, mode, k, density, &P)) return SEER_ERR_INVALID_ARG;
  if (!dbuf || !aligned(dbuf, 256) || dbuf_bytes < P.total) return SEER_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t perr = cudaSuccess;
  HostPipe* pp = host_pipe(&perr);
  if (!pp) return cuda_fail(perr);
  HostPipe& pipe = *pp;
  // the copy streams start after the work already queued on the caller's stream
  SEER_CUDA(cudaEventRecord(pipe.start, st));
  SEER_CUDA(cudaStreamWaitEvent(pipe.in, pipe.start, 0));
  SEER_CUDA(cudaStreamWaitEvent(pipe.out, pipe.start, 0));
  uint8_t* const base = (uint8_t*)dbuf;
  uint32_t* const status = (uint32_t*)(base + P.status);
  SEER_CUDA(cudaMemsetAsync(status, 0, sizeof(uint32_t) * 2 * (size_t)P.chunks, st));
  const size_t n = (size_t)dims->n, d = (size_t)dims->d, es = dtype == SEER_FP32 ? 4 : 2;
  const int Hq = dims->Hq, Hkv = dims->Hkv, G = P.G, C = P.C;
  seer_status err = SEER_OK;
  for (int i = 0; i < P.chunks && err == SEER_OK; ++i) {
    const int kvi = i / P.per_kv, part = i % P.per_kv;  // KV head (b*Hkv + g) and chunk within it
    const int b = kvi / Hkv, g = kvi % Hkv, s = i % kHostSlots, t = kvi % kHostSlots;
    const int hq0 = g * G + part * C;  // first query head of the chunk
    uint8_t* const slot = base + (size_t)s * P.slot;
    uint8_t* const kvs = base + P.kv_base + (size_t)t * P.kvslot;
    const size_t q_off = ((size_t)b * Hq + hq0) * n * d * es;
    const size_t kv_off = ((size_t)b * Hkv + g) * n * d * es;
    if (part == 0) {
      // K and V of this KV head, once its slot's previous KV head is done
      if (kvi >= kHostSlots) SEER_CUDA(cudaStreamWaitEvent(pipe.in, pipe.kv_done[t], 0));
      SEER_CUDA(cudaMemcpyAsync(kvs + P.s_k, (const uint8_t*)hK + kv_off, P.kv, cudaMemcpyHostToDevice, pipe.in));
      SEER_CUDA(cudaMemcpyAsync(kvs + P.s_v, (const uint8_t*)hV + kv_off, P.kv, cudaMemcpyHostToDevice, pipe.in));
      SEER_CUDA(cudaEventRecord(pipe.kv_in[t], pipe.in));
    }
    // the chunk slot's Q is free once the compute two chunks back is done
    if (i >= kHostSlots) SEER_CUDA(cudaStreamWaitEvent(pipe.in, pipe.computed[s], 0));
    SEER_CUDA(cudaMemcpyAsync(slot + P.s_q, (const uint8_t*)hQ + q_off, P.q, cudaMemcpyHostToDevice, pipe.in));
    SEER_CUDA(cudaEventRecord(pipe.copied_in[s], pipe.in));
    // compute: after the copies in, and once the copy out two chunks back
    // has released the slot's O, LSE and lists
    SEER_CUDA(cudaStreamWaitEvent(st, pipe.copied_in[s], 0));
    SEER_CUDA(cudaStreamWaitEvent(st, pipe.kv_in[t], 0));
    if (i >= kHostSlots) SEER_CUDA(cudaStreamWaitEvent(st, pipe.copied_out[s], 0));
    int32_t* const cnt = (int32_t*)(slot + P.s_cnt);
    int32_t* const idx = (int32_t*)(slot + P.s_idx);
    err = seer_gate(&P.g, slot + P.s_q, kvs + P.s_k, dtype, Wq + (size_t)hq0 * h * d, Wk + (size_t)g * h * 3 * d,
                    h, rope_theta, mode, T, k, density, nullptr, cnt, idx, P.cap, base + P.gate_ws,
                    P.gate_ws_bytes, stream);
    if (err != SEER_OK) break;
    SEER_CUDA(cudaMemcpyAsync(status + 2 * i, base + P.gate_ws, sizeof(uint32_t), cudaMemcpyDeviceToDevice, st));
    err = seer_sparse_attn(&P.g, slot + P.s_q, kvs + P.s_k, kvs + P.s_v, dtype, cnt, idx, P.cap, scale,
                           slot + P.s_o, hLSE ? (float*)(slot + P.s_lse) : nullptr, base + P.attn_ws,
                           P.attn_ws_bytes, stream);
    if (err != SEER_OK) break;
    SEER_CUDA(cudaMemcpyAsync(status + 2 * i + 1, base + P.attn_ws, sizeof(uint32_t), cudaMemcpyDeviceToDevice, st));
    SEER_CUDA(cudaEventRecord(pipe.computed[s], st));
    if (part == P.per_kv - 1) SEER_CUDA(cudaEventRecord(pipe.kv_done[t], st));
    // out
    SEER_CUDA(cudaStreamWaitEvent(pipe.out, pipe.computed[s], 0));
    SEER_CUDA(cudaMemcpyAsync((uint8_t*)hO + q_off, slot + P.s_o, P.o, cudaMemcpyDeviceToHost, pipe.out));
    if (hLSE)
      SEER_CUDA(cudaMemcpyAsync(hLSE + ((size_t)b * Hq + hq0) * n, slot + P.s_lse, P.lse, cudaMemcpyDeviceToHost,
                                pipe.out));
    SEER_CUDA(cudaEventRecord(pipe.copied_out[s], pipe.out));
  }
  // the caller's stream ends after the last copy out (the copy-out stream is
  // in order) and after every copy in
  SEER_CUDA(cudaEventRecord(pipe.start, pipe.out));
  SEER_CUDA(cudaStreamWaitEvent(st, pipe.start, 0));
  SEER_CUDA(cudaEventRecord(pipe.start, pipe.in));
  SEER_CUDA(cudaStreamWaitEvent(st, pipe.start, 0));
  if (err != SEER_OK) {
    cudaStreamSynchronize(st);
    return err;
  }
  std::vector<uint32_t> words(2 * (size_t)P.chunks);
  SEER_CUDA(cudaMemcpyAsync(words.data(), status, sizeof(uint32_t) * words.size(), cudaMemcpyDeviceToHost, st));
  SEER_CUDA(cudaStreamSynchronize(st));
  for (uint32_t w : words)
    if (w == seer::kDevTimeout) return SEER_ERR_TIMEOUT;
  for (uint32_t w : words)
    if (w != seer::kDevOk) return SEER_ERR_DEVICE_CHECK;
  return SEER_OK;
}

}  // extern "C"
