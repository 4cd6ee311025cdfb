// C-ABI entry points of libkvrq.so: argument validation (host, before any
// launch), TMA tensor-map encoding, kernel dispatch and status reporting.

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "kvrq.h"
#include "kvrq_internal.h"
#include "rq_launch.h"
#include "tq_launch.h"
#include "tqg_launch.h"
#include "score_launch.h"
#include "attn_launch.h"
#include "pq_launch.h"

namespace kvrq {

// Device status word (see kvrq_device_status); one per device image.
__device__ unsigned int g_device_status = 0;

static thread_local std::string t_last_error;

// Allocation failures the test hook still has to inject (kvrq_test_fail_allocations).
static std::atomic<int> g_fail_allocs{0};

// Polls after which the packed-score kernel's main-loop waits give up (kvrq_set_wait_limit; < 0: default).
static std::atomic<int32_t> g_wait_limit{-1};

void alloc_check() {
  int left = g_fail_allocs.load();
  while (left > 0) {
    if (g_fail_allocs.compare_exchange_weak(left, left - 1)) throw std::bad_alloc();
  }
}

kvrq_status set_error(kvrq_status st, const char* msg) {
  t_last_error = msg ? msg : "";
  return st;
}

kvrq_status set_errorf(kvrq_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return st;
}

static kvrq_status cuda_fail(const char* where, cudaError_t e) {
  return set_errorf(KVRQ_ECUDA, "%s: %s", where, cudaGetErrorString(e));
}

// ------------------------------------------------------------------ per-device state
// Scratch of tq_quantize_prod_noalloc: one per device image, 8 MiB. Nothing in
// it has to start at zero (each call writes every byte it later reads), and
// calls that overlap in time on one device share it, so they race.
constexpr size_t kNoallocScratchBytes = (size_t)8 << 20;
static __device__ __align__(256) unsigned char g_tq_scratch[kNoallocScratchBytes];

constexpr int kHostSlots = 3;  // chunks in flight in the host-buffer pipeline

struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  unsigned* status = nullptr;  // device address of g_device_status
  void* scratch = nullptr;     // device address of g_tq_scratch
  // host-buffer pipeline (created at its first call): copy-in, compute and copy-out streams,
  // per-slot events, the start and end events of a call, and a lock that keeps one call's
  // issue sequence whole
  bool pipe_ready = false;
  cudaStream_t pipe[3] = {nullptr, nullptr, nullptr};
  cudaEvent_t in_done[kHostSlots] = {}, comp_done[kHostSlots] = {}, out_done[kHostSlots] = {};
  cudaEvent_t ev_start = nullptr, ev_end = nullptr;
  std::mutex pipe_mu;
};

static std::mutex g_dev_mu;
static DeviceInfo g_dev[64];

static kvrq_status current_device(DeviceInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
  if (dev < 0 || dev >= 64) return set_error(KVRQ_EUNSUPPORTED, "device ordinal >= 64");
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.ready) {
    e = cudaDeviceGetAttribute(&di.num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail("cudaDeviceGetAttribute", e);
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_device_status);
    if (e != cudaSuccess) return cuda_fail("cudaGetSymbolAddress(status)", e);
    di.status = static_cast<unsigned*>(p);
    e = cudaGetSymbolAddress(&p, g_tq_scratch);
    if (e != cudaSuccess) return cuda_fail("cudaGetSymbolAddress(scratch)", e);
    di.scratch = p;
    di.ready = true;
  }
  *out = &di;
  return KVRQ_OK;
}

// ------------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static kvrq_status get_encode(EncodeTiledFn* fn) {
  static EncodeTiledFn cached = nullptr;
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess) cached = reinterpret_cast<EncodeTiledFn>(p);
  });
  if (!cached) return set_error(KVRQ_ECUDA, "cuTensorMapEncodeTiled is not available from the driver");
  *fn = cached;
  return KVRQ_OK;
}

static size_t dtype_size(kvrq_dtype t) { return t == KVRQ_F32 ? 4 : 2; }

static CUtensorMapDataType tma_type(kvrq_dtype t) {
  return t == KVRQ_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                       : (t == KVRQ_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}

// Row-major [rows][ld] matrix, first `cols` columns, boxes of 128 bytes x box_rows,
// 128-byte swizzle, zero fill out of range.
kvrq_status encode_rows_map(CUtensorMap* map, const void* ptr, kvrq_dtype dt, int64_t rows, int64_t cols, int64_t ld,
                            int box_rows) {
  EncodeTiledFn enc;
  kvrq_status st = get_encode(&enc);
  if (st != KVRQ_OK) return st;
  const size_t es = dtype_size(dt);
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * es)};
  cuuint32_t box[2] = {(cuuint32_t)(128 / es), (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, tma_type(dt), 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_errorf(KVRQ_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return KVRQ_OK;
}

// ------------------------------------------------------------------ validation helpers
static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static bool valid_dtype(int t) { return t == KVRQ_F32 || t == KVRQ_F16 || t == KVRQ_BF16; }

// Rows of a [n][ld] matrix start 16-byte aligned.
static bool rows_aligned16(const void* p, int64_t ld, kvrq_dtype dt) {
  return aligned(p, 16) && ((ld * (int64_t)dtype_size(dt)) % 16) == 0;
}

static kvrq_status launch_status(const char* where, cudaError_t e) {
  if (e != cudaSuccess) return cuda_fail(where, e);
  return KVRQ_OK;
}

// Shared validation and dispatch of the three RotorQuant calls.
static kvrq_status rq_call(const char* name, int mode, void* stream, const void* x, kvrq_dtype xdt, int64_t ldx,
                           const uint32_t* codes_in, uint32_t* codes_out, int64_t ldc, const float* norms_in,
                           float* norms_out, int64_t n, int d, const float* rotors, const float* centroids, int bits,
                           void* xhat, kvrq_dtype odt, int64_t ldo, int64_t ldn = 1, int cpg = 3,
                           const int64_t* out_rows = nullptr) {
  if (ldn < 1) return set_errorf(KVRQ_EINVAL, "%s: norm row stride < 1", name);
  if (n < 0) return set_errorf(KVRQ_EINVAL, "%s: n < 0", name);
  if (d < 2 || d > (1 << 20)) return set_errorf(KVRQ_EINVAL, "%s: d must be in 2..2^20", name);
  if (bits < 1 || bits > 4) return set_errorf(KVRQ_EUNSUPPORTED, "%s: bits must be in 1..4", name);
  const bool q_side = mode != RQ_DQ, dq_side = mode != RQ_Q;
  if (q_side && !valid_dtype(xdt)) return set_errorf(KVRQ_EINVAL, "%s: bad input dtype", name);
  if (dq_side && !valid_dtype(odt)) return set_errorf(KVRQ_EINVAL, "%s: bad output dtype", name);
  const int G = (d + 2) / 3;
  const int64_t W = kvrq_packed_words(cpg * (int64_t)G, bits);
  if (cpg == 4 && d != 128) return set_errorf(KVRQ_EUNSUPPORTED, "%s: the four-grade layout takes d = 128", name);
  if (n == 0) return KVRQ_OK;
  if (!rotors || !centroids) return set_errorf(KVRQ_EINVAL, "%s: rotors and centroids are required", name);
  if (!aligned(rotors, 16) || !aligned(centroids, 4))
    return set_errorf(KVRQ_EINVAL, "%s: rotors must be 16-byte aligned, centroids 4-byte aligned", name);
  if (q_side) {
    if (!x) return set_errorf(KVRQ_EINVAL, "%s: x is NULL", name);
    if (ldx < d) return set_errorf(KVRQ_EINVAL, "%s: ldx < d", name);
    if (!aligned(x, dtype_size(xdt))) return set_errorf(KVRQ_EINVAL, "%s: x misaligned", name);
    if (mode == RQ_Q && (!codes_out || !norms_out)) return set_errorf(KVRQ_EINVAL, "%s: codes and norms are required", name);
    if (codes_out && (ldc < W || !aligned(codes_out, 4))) return set_errorf(KVRQ_EINVAL, "%s: ldc < packed words or codes misaligned", name);
    if (norms_out && !aligned(norms_out, 4)) return set_errorf(KVRQ_EINVAL, "%s: norms misaligned", name);
  } else {
    if (!codes_in || !norms_in) return set_errorf(KVRQ_EINVAL, "%s: codes and norms are required", name);
    if (ldc < W || !aligned(codes_in, 4) || !aligned(norms_in, 4))
      return set_errorf(KVRQ_EINVAL, "%s: ldc < packed words or codes/norms misaligned", name);
  }
  if (dq_side) {
    if (!xhat) return set_errorf(KVRQ_EINVAL, "%s: xhat is NULL", name);
    if (ldo < d) return set_errorf(KVRQ_EINVAL, "%s: ldo < d", name);
    if (!aligned(xhat, dtype_size(odt))) return set_errorf(KVRQ_EINVAL, "%s: xhat misaligned", name);
  }
  if (n > ((int64_t)1 << 31) - 256) return set_errorf(KVRQ_EUNSUPPORTED, "%s: n >= 2^31", name);
  if (out_rows && !(mode == RQ_Q && d == 128 && rows_aligned16(x, ldx, xdt)))
    return set_errorf(KVRQ_EUNSUPPORTED, "%s: destination rows need d = 128 and 16-byte aligned rows", name);

  DeviceInfo* di;
  kvrq_status st = current_device(&di);
  if (st != KVRQ_OK) return st;
  RqArgs a{};
  a.n = n;
  a.d = d;
  a.rotors = rotors;
  a.centroids = centroids;
  a.x = x;
  a.ldx = ldx;
  a.codes_out = codes_out;
  a.norms_out = norms_out;
  a.codes_in = codes_in;
  a.norms_in = norms_in;
  a.xhat = xhat;
  a.ldo = ldo;
  a.ldc = ldc;
  a.ldn = ldn;
  a.status = di->status;
  a.codes_per_group = cpg;
  a.out_rows = out_rows;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  const kvrq_dtype tdt = q_side ? xdt : odt;
  bool row_path = rq_row_dims(d, xdt) && rq_row_dims(d, odt);
  if (q_side) row_path = row_path && rows_aligned16(x, ldx, xdt);
  if (dq_side) row_path = row_path && rows_aligned16(xhat, ldo, odt);
  if (mode == RQ_QDQ) row_path = row_path && xdt == odt;
  if (row_path) {
    CUtensorMap mx, mo;
    memset(&mx, 0, sizeof(mx));
    memset(&mo, 0, sizeof(mo));
    if (q_side && (st = encode_rows_map(&mx, x, xdt, n, d, ldx, rq_row_box_rows())) != KVRQ_OK) return st;
    if (dq_side && (st = encode_rows_map(&mo, xhat, odt, n, d, ldo, rq_row_box_rows())) != KVRQ_OK) return st;
    if (!q_side) mx = mo;
    if (!dq_side) mo = mx;
    return launch_status(name, launch_rq_row(mode, tdt, bits, mx, mo, a, s, di->num_sms));
  }
  if (cpg == 4)
    return set_errorf(KVRQ_EUNSUPPORTED, "%s: the four-grade layout needs 16-byte aligned rows (and one dtype for "
                                         "the fused call)", name);

  // any d: rows streamed by bulk copy when they start 16-byte aligned and fit its row buffers
  bool wide = true;
  if (q_side) wide = wide && rows_aligned16(x, ldx, xdt);
  if (dq_side) wide = wide && rows_aligned16(xhat, ldo, odt);
  if (mode == RQ_QDQ) wide = wide && xdt == odt;
  a.wide = wide && rq_wide_smem_bytes(d, bits, (int)dtype_size(tdt)) > 0;
  return launch_status(name, launch_rq_general(mode, xdt, odt, bits, a, s, di->num_sms));
}


static int tile_n(int n_total) { return n_total % 256 == 0 ? 256 : 128; }

static size_t tq_ws_row_bytes(int d) { return (size_t)4 * d + (size_t)4 * (d / 128); }

// Tiled TurboQuant path (tqg_kernels.cu): every d that is a multiple of 128,
// fp32 vectors included. Arguments are validated by tq_call.
static kvrq_status tqg_call(const char* name, int mode, cudaStream_t s, DeviceInfo* di, const void* x, kvrq_dtype dt,
                            int64_t ldx, int64_t n, int d, int m, const void* pi, const uint16_t* T,
                            const float* centroids, int cbits, uint32_t* codes_out, const uint32_t* codes_in,
                            int64_t ldc, uint32_t* signs_out, const uint32_t* signs_in, int64_t lds,
                            float* gammas_out, const float* gammas_in, float* norms_out, const float* norms_in,
                            void* xhat, int64_t ldo, int64_t ldn, void* ws, size_t ws_bytes) {
  const bool f32 = dt == KVRQ_F32;
  const kvrq_dtype pdt = f32 ? KVRQ_F16 : dt;  // operand type of Pi
  const int bn_d = tile_n(d), bn_m = tile_n(m);
  kvrq_status st;
  CUtensorMap none, mx, mo;
  memset(&none, 0, sizeof(none));
  memset(&mx, 0, sizeof(mx));
  memset(&mo, 0, sizeof(mo));
  TqgArgs base{};
  base.d = d;
  base.n_part = d / bn_d;
  base.centroids = centroids;
  base.qjl_scale = (float)(1.2533141373155003 / (double)m);  // sqrt(pi/2) / m
  base.ldx = ldx;
  base.ldc = ldc;
  base.lds = lds;
  base.ldn = ldn;
  base.status = di->status;
  const bool q_side = mode == TQ_MSE_Q || mode == TQ_MSE_QDQ || mode == TQ_PROD_Q;
  const bool out = mode == TQ_MSE_QDQ || mode == TQ_DQ_MSE || mode == TQ_DQ_PROD;
  if (q_side && !f32 && (st = encode_rows_map(&mx, x, dt, n, d, ldx, 128)) != KVRQ_OK) return st;
  if (out && (st = encode_rows_map(&mo, xhat, dt, n, d, ldo, 128)) != KVRQ_OK) return st;
  auto launch = [&](int gmode, int bn, const CUtensorMap& ma, const CUtensorMap& mb, const TqgArgs& a) {
    return launch_status(name, launch_tqg(gmode, dt, cbits, bn, ma, mb, mo, a, s, di->num_sms));
  };

  if (mode == TQ_MSE_Q || mode == TQ_MSE_QDQ || mode == TQ_DQ_MSE) {
    if (mode != TQ_DQ_MSE) {
      CUtensorMap mp;
      if ((st = encode_rows_map(&mp, pi, pdt, d, d, d, bn_d)) != KVRQ_OK) return st;
      TqgArgs a = base;
      a.n = n;
      a.k_total = d;
      a.n_total = d;
      a.xf = f32 ? static_cast<const float*>(x) : nullptr;
      a.codes_out = codes_out;
      a.norms_out = norms_out;
      if ((st = launch(G_MSE_Q, bn_d, mx, mp, a)) != KVRQ_OK) return st;
    }
    if (mode != TQ_MSE_Q) {
      CUtensorMap mpt;
      if ((st = encode_rows_map(&mpt, pi, pdt, d, d, d, 64)) != KVRQ_OK) return st;
      TqgArgs a = base;
      a.n = n;
      a.k_total = d;
      a.n_total = d;
      a.codes_in = mode == TQ_DQ_MSE ? codes_in : codes_out;
      a.norms_in = mode == TQ_DQ_MSE ? norms_in : norms_out;
      if ((st = launch(G_DQ_MSE, bn_d, none, mpt, a)) != KVRQ_OK) return st;
    }
    return KVRQ_OK;
  }

  // prod: blocks of rows through the workspace
  const int64_t cap = (int64_t)(ws_bytes / tq_ws_row_bytes(d)) / 128 * 128;
  if (!ws || cap < 128)
    return set_errorf(KVRQ_EINVAL, "%s: workspace of %zu bytes holds fewer than 128 rows (need %zu per row)", name,
                      ws_bytes, tq_ws_row_bytes(d));
  if (!aligned(ws, 16)) return set_errorf(KVRQ_EINVAL, "%s: workspace must be 16-byte aligned", name);
  float* part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + (size_t)cap * 4 * d);
  if (mode == TQ_PROD_Q) {
    CUtensorMap mp, mt, mr;
    if ((st = encode_rows_map(&mp, pi, pdt, d, d, d, bn_d)) != KVRQ_OK) return st;
    if ((st = encode_rows_map(&mt, T, KVRQ_F16, m, d, d, bn_m)) != KVRQ_OK) return st;
    if ((st = encode_rows_map(&mr, ws, KVRQ_F16, cap, d, d, 128)) != KVRQ_OK) return st;
    for (int64_t r0 = 0; r0 < n; r0 += cap) {
      const int64_t rows = n - r0 < cap ? n - r0 : cap;
      TqgArgs a = base;
      a.n = rows;
      a.k_total = d;
      a.n_total = d;
      a.map_row0 = r0;
      a.xf = f32 ? static_cast<const float*>(x) + r0 * ldx : nullptr;
      a.codes_out = codes_out + r0 * ldc;
      a.norms_out = norms_out + r0 * ldn;
      a.ws = ws;
      a.part = part;
      if ((st = launch(G_PROD_Q1, bn_d, mx, mp, a)) != KVRQ_OK) return st;
      TqgArgs b = base;
      b.n = rows;
      b.k_total = d;
      b.n_total = m;
      b.signs_out = signs_out + r0 * lds;
      b.gammas_out = gammas_out + r0 * ldn;
      b.part = part;
      if ((st = launch(G_PROD_Q2, bn_m, mr, mt, b)) != KVRQ_OK) return st;
    }
    return KVRQ_OK;
  }
  // TQ_DQ_PROD
  CUtensorMap mtt, mpt, mw;
  memset(&mw, 0, sizeof(mw));
  if ((st = encode_rows_map(&mtt, T, KVRQ_F16, m, d, d, 64)) != KVRQ_OK) return st;
  if ((st = encode_rows_map(&mpt, pi, pdt, d, d, d, 64)) != KVRQ_OK) return st;
  if (!f32 && (st = encode_rows_map(&mw, ws, dt, cap, d, d, 128)) != KVRQ_OK) return st;
  for (int64_t r0 = 0; r0 < n; r0 += cap) {
    const int64_t rows = n - r0 < cap ? n - r0 : cap;
    TqgArgs a = base;
    a.n = rows;
    a.k_total = m;
    a.n_total = d;
    a.codes_in = codes_in + r0 * ldc;
    a.signs_in = signs_in + r0 * lds;
    a.gammas_in = gammas_in + r0 * ldn;
    a.ws = ws;
    if ((st = launch(G_DQ_PROD1, bn_d, none, mtt, a)) != KVRQ_OK) return st;
    TqgArgs b = base;
    b.n = rows;
    b.k_total = d;
    b.n_total = d;
    b.map_row0 = r0;
    b.norms_in = norms_in + r0 * ldn;
    b.ws = ws;
    if ((st = launch(G_DQ_PROD2, bn_d, mw, mpt, b)) != KVRQ_OK) return st;
  }
  return KVRQ_OK;
}

// Shared validation and dispatch of the TurboQuant calls: d = m = 128 with
// fp16/bf16 vectors on the resident-Pi kernels, everything else (d a multiple
// of 128, fp32 vectors) on the tiled kernel.
static kvrq_status tq_call(const char* name, int mode, void* stream, const void* x, kvrq_dtype dt, int64_t ldx,
                           int64_t n, int d, int m, const void* pi, const uint16_t* T, const float* centroids,
                           int bits, uint32_t* codes_out, const uint32_t* codes_in, int64_t ldc, uint32_t* signs_out,
                           const uint32_t* signs_in, int64_t lds, float* gammas_out, const float* gammas_in,
                           float* norms_out, const float* norms_in, void* xhat, int64_t ldo, int64_t ldn = 1,
                           void* ws = nullptr, size_t ws_bytes = 0, bool static_scratch = false,
                           const int64_t* out_rows = nullptr) {
  const bool prod = mode == TQ_PROD_Q || mode == TQ_DQ_PROD;
  if (ldn < 1) return set_errorf(KVRQ_EINVAL, "%s: norm row stride < 1", name);
  const bool q_side = mode == TQ_MSE_Q || mode == TQ_MSE_QDQ || mode == TQ_PROD_Q;
  const bool out = mode == TQ_MSE_QDQ || mode == TQ_DQ_MSE || mode == TQ_DQ_PROD;
  if (n < 0) return set_errorf(KVRQ_EINVAL, "%s: n < 0", name);
  if (d < 2) return set_errorf(KVRQ_EINVAL, "%s: d must be >= 2", name);
  if (!valid_dtype(dt)) return set_errorf(KVRQ_EINVAL, "%s: bad dtype", name);
  if (prod ? (bits < 2 || bits > 5) : (bits < 1 || bits > 4))
    return set_errorf(KVRQ_EUNSUPPORTED, "%s: bits must be in %s", name, prod ? "2..5" : "1..4");
  if (d % 128 != 0 || d > 16384)
    return set_errorf(KVRQ_EUNSUPPORTED, "%s: the tensor-core paths need d a multiple of 128 (<= 16384)", name);
  if (prod && m != d) return set_errorf(KVRQ_EUNSUPPORTED, "%s: the QJL projection needs m = d", name);
  const bool tiled = d != 128 || dt == KVRQ_F32;
  if (out_rows && tiled)
    return set_errorf(KVRQ_EUNSUPPORTED, "%s: destination rows need d = 128 and fp16 or bf16 vectors", name);
  const int cbits = prod ? bits - 1 : bits;
  const int64_t W = kvrq_packed_words(d, cbits);
  if (n == 0) return KVRQ_OK;
  if (!pi || !centroids || (prod && !T)) return set_errorf(KVRQ_EINVAL, "%s: pi, centroids (and T) are required", name);
  if (!aligned(pi, 16) || (T && !aligned(T, 16)) || !aligned(centroids, 4))
    return set_errorf(KVRQ_EINVAL, "%s: pi and T must be 16-byte aligned", name);
  if (q_side) {
    if (!x || ldx < d || !rows_aligned16(x, ldx, dt)) return set_errorf(KVRQ_EINVAL, "%s: x NULL, ldx < d or rows not 16-byte aligned", name);
    if ((tiled || mode != TQ_MSE_QDQ) && (!codes_out || !norms_out))
      return set_errorf(KVRQ_EINVAL, "%s: codes and norms are required", name);
    if (codes_out && (ldc < W || !aligned(codes_out, 4))) return set_errorf(KVRQ_EINVAL, "%s: ldc < packed words", name);
    if (prod && (!signs_out || !gammas_out || lds < m / 32 || !aligned(signs_out, 4)))
      return set_errorf(KVRQ_EINVAL, "%s: signs (lds >= m/32) and gammas are required", name);
  } else {
    if (!codes_in || !norms_in || ldc < W) return set_errorf(KVRQ_EINVAL, "%s: codes, norms (ldc >= packed words) are required", name);
    if (prod && (!signs_in || !gammas_in || lds < m / 32)) return set_errorf(KVRQ_EINVAL, "%s: signs and gammas are required", name);
  }
  if (out && (!xhat || ldo < d || !rows_aligned16(xhat, ldo, dt)))
    return set_errorf(KVRQ_EINVAL, "%s: xhat NULL, ldo < d or rows not 16-byte aligned", name);
  if (n > ((int64_t)1 << 31) - 256) return set_errorf(KVRQ_EUNSUPPORTED, "%s: n >= 2^31", name);
  if (tiled && prod && static_scratch && 128 * tq_ws_row_bytes(d) > kNoallocScratchBytes)
    return set_errorf(KVRQ_EUNSUPPORTED,
                      "%s: d = %d needs %zu bytes of scratch for one 128-row block; the static scratch holds %zu",
                      name, d, 128 * tq_ws_row_bytes(d), kNoallocScratchBytes);
  if (tiled && prod && !static_scratch && (!ws || ws_bytes / tq_ws_row_bytes(d) < 128 || !aligned(ws, 16)))
    return set_errorf(KVRQ_EINVAL, "%s: workspace (16-byte aligned) of %zu bytes holds fewer than 128 rows (need %zu per row)",
                      name, ws_bytes, tq_ws_row_bytes(d));

  DeviceInfo* di;
  kvrq_status st = current_device(&di);
  if (st != KVRQ_OK) return st;
  if (static_scratch) {
    ws = di->scratch;
    ws_bytes = kNoallocScratchBytes;
  }
  if (tiled)
    return tqg_call(name, mode, static_cast<cudaStream_t>(stream), di, x, dt, ldx, n, d, m, pi, T, centroids, cbits,
                    codes_out, codes_in, ldc, signs_out, signs_in, lds, gammas_out, gammas_in, norms_out, norms_in,
                    xhat, ldo, ldn, ws, ws_bytes);
  CUtensorMap mx, mp, mt, mo;
  memset(&mx, 0, sizeof(mx));
  memset(&mp, 0, sizeof(mp));
  memset(&mt, 0, sizeof(mt));
  memset(&mo, 0, sizeof(mo));
  if ((st = encode_rows_map(&mp, pi, dt, d, d, d, 128)) != KVRQ_OK) return st;
  if (prod && (st = encode_rows_map(&mt, T, KVRQ_F16, m, d, d, 128)) != KVRQ_OK) return st;
  if (q_side && (st = encode_rows_map(&mx, x, dt, n, d, ldx, 128)) != KVRQ_OK) return st;
  if (out && (st = encode_rows_map(&mo, xhat, dt, n, d, ldo, 128)) != KVRQ_OK) return st;
  TqArgs a{};
  a.n = n;
  a.d = d;
  a.centroids = centroids;
  a.qjl_scale = (float)(1.2533141373155003 / (double)m);  // sqrt(pi/2) / m
  a.ldx = ldx;
  a.codes_out = codes_out;
  a.norms_out = norms_out;
  a.signs_out = signs_out;
  a.gammas_out = gammas_out;
  a.codes_in = codes_in;
  a.norms_in = norms_in;
  a.signs_in = signs_in;
  a.gammas_in = gammas_in;
  a.ldc = ldc;
  a.lds = lds;
  a.ldn = ldn;
  a.status = di->status;
  a.out_rows = out_rows;
  return launch_status(name, launch_tq(mode, dt, cbits, mx, mp, mt, mo, a, static_cast<cudaStream_t>(stream), di->num_sms));
}

// PolarQuant at d = 128 (fused roundtrip, or dequantize of stored code rows).
static kvrq_status pq_call(const char* name, int mode, void* stream, const void* x, kvrq_dtype dt, int64_t ldx,
                           int64_t n, int d, const void* pi, const float* centroids, uint32_t* codes_out,
                           const uint32_t* codes_in, int64_t ldc, void* xhat, int64_t ldo) {
  if (n < 0) return set_errorf(KVRQ_EINVAL, "%s: n < 0", name);
  if (d != 128) return set_errorf(KVRQ_EUNSUPPORTED, "%s: d = 128 is supported (four levels of 4, 2, 2, 2 bits)", name);
  if (dt != KVRQ_F16 && dt != KVRQ_BF16) return set_errorf(KVRQ_EUNSUPPORTED, "%s: fp16 or bf16 vectors", name);
  if (n == 0) return KVRQ_OK;
  if (!pi || !aligned(pi, 16) || !centroids || !aligned(centroids, 4))
    return set_errorf(KVRQ_EINVAL, "%s: pi (16-byte aligned) and centroids are required", name);
  if (mode == PQ_QDQ && (!x || ldx < d || !rows_aligned16(x, ldx, dt)))
    return set_errorf(KVRQ_EINVAL, "%s: x NULL, ldx < d or rows not 16-byte aligned", name);
  if (mode == PQ_DQ && !codes_in) return set_errorf(KVRQ_EINVAL, "%s: codes are required", name);
  if ((codes_in || codes_out) && (ldc < kPqWords || !aligned(codes_in ? (const void*)codes_in : codes_out, 4)))
    return set_errorf(KVRQ_EINVAL, "%s: ldc must be >= %d code words", name, kPqWords);
  if (!xhat || ldo < d || !rows_aligned16(xhat, ldo, dt))
    return set_errorf(KVRQ_EINVAL, "%s: xhat NULL, ldo < d or rows not 16-byte aligned", name);
  if (n > ((int64_t)1 << 31) - 256) return set_errorf(KVRQ_EUNSUPPORTED, "%s: n >= 2^31", name);
  DeviceInfo* di;
  kvrq_status st = current_device(&di);
  if (st != KVRQ_OK) return st;
  CUtensorMap mx, mp, mo;
  memset(&mx, 0, sizeof(mx));
  memset(&mp, 0, sizeof(mp));
  memset(&mo, 0, sizeof(mo));
  if ((st = encode_rows_map(&mp, pi, dt, d, d, d, 128)) != KVRQ_OK) return st;
  if (mode == PQ_QDQ && (st = encode_rows_map(&mx, x, dt, n, d, ldx, 128)) != KVRQ_OK) return st;
  if ((st = encode_rows_map(&mo, xhat, dt, n, d, ldo, 128)) != KVRQ_OK) return st;
  if (mode != PQ_QDQ) mx = mo;
  PqArgs a{};
  a.n = n;
  a.centroids = centroids;
  a.codes_out = codes_out;
  a.codes_in = codes_in;
  a.ldc = ldc;
  a.status = di->status;
  return launch_status(name, launch_pq(mode, dt, mx, mp, mo, a, static_cast<cudaStream_t>(stream), di->num_sms));
}

// The QJL sign sketch of arbitrary rows (tiled kernel, sketch epilogue).
static kvrq_status qjl_call(void* stream, const void* r, kvrq_dtype dt, int64_t n, int d, int64_t ldr, const void* T,
                            int m, uint32_t* signs, int64_t lds, float* gammas, int64_t ldn) {
  const char* name = "qjl_sketch";
  if (n < 0 || ldn < 1) return set_errorf(KVRQ_EINVAL, "%s: n < 0 or ldn < 1", name);
  if (!valid_dtype(dt)) return set_errorf(KVRQ_EINVAL, "%s: bad dtype", name);
  if (d < 64 || d % 64 != 0 || d > 16384 || m < 128 || m % 128 != 0)
    return set_errorf(KVRQ_EUNSUPPORTED, "%s: d must be a multiple of 64 (<= 16384) and m a multiple of 128", name);
  if (n == 0) return KVRQ_OK;
  if (!r || ldr < d || !rows_aligned16(r, ldr, dt)) return set_errorf(KVRQ_EINVAL, "%s: r NULL, ldr < d or rows not 16-byte aligned", name);
  if (!T || !aligned(T, 16)) return set_errorf(KVRQ_EINVAL, "%s: T must be a 16-byte aligned pointer", name);
  if (!signs || lds < m / 32 || !aligned(signs, 4) || !gammas)
    return set_errorf(KVRQ_EINVAL, "%s: signs (lds >= m/32) and gammas are required", name);
  if (n > ((int64_t)1 << 31) - 256) return set_errorf(KVRQ_EUNSUPPORTED, "%s: n >= 2^31", name);
  DeviceInfo* di;
  kvrq_status st = current_device(&di);
  if (st != KVRQ_OK) return st;
  const bool f32 = dt == KVRQ_F32;
  const int bn = tile_n(m);
  CUtensorMap mr, mt, none;
  memset(&mr, 0, sizeof(mr));
  memset(&none, 0, sizeof(none));
  if (!f32 && (st = encode_rows_map(&mr, r, dt, n, d, ldr, 128)) != KVRQ_OK) return st;
  if ((st = encode_rows_map(&mt, T, f32 ? KVRQ_F16 : dt, m, d, d, bn)) != KVRQ_OK) return st;
  TqgArgs a{};
  a.n = n;
  a.d = d;
  a.k_total = d;
  a.n_total = m;
  a.xf = f32 ? static_cast<const float*>(r) : nullptr;
  a.ldx = ldr;
  a.signs_out = signs;
  a.lds = lds;
  a.gammas_out = gammas;
  a.ldn = ldn;
  a.status = di->status;
  return launch_status(name, launch_tqg(G_SKETCH, dt, 1, bn, mr, mt, none, a, static_cast<cudaStream_t>(stream),
                                        di->num_sms));
}

}  // namespace kvrq

using namespace kvrq;

extern "C" {

const char* kvrq_version(void) { return "kvrq 0.1.0 (sm_100a)"; }

const char* kvrq_last_error_string(void) { return t_last_error.c_str(); }

kvrq_status kvrq_device_status(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned h = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&h, g_device_status, sizeof(h), 0, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail("kvrq_device_status", e);
  if (h & 1u) return set_error(KVRQ_ETIMEOUT, "a bounded device-side wait ran out");
  if (h) return set_errorf(KVRQ_ECUDA, "device status word 0x%x", h);
  return KVRQ_OK;
}

kvrq_status rq_quantize(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d, int64_t ldx,
                        const float* rotors, const float* centroids, int bits, uint32_t* codes, int64_t ldc,
                        float* norms) {
  return rq_call("rq_quantize", RQ_Q, stream, x, xdtype, ldx, nullptr, codes, ldc, nullptr, norms, n, d, rotors,
                 centroids, bits, nullptr, xdtype, 0);
}

kvrq_status rq_dequantize(void* stream, const uint32_t* codes, int64_t ldc, const float* norms, int64_t n, int d,
                          const float* rotors, const float* centroids, int bits, void* xhat, kvrq_dtype odtype,
                          int64_t ldo) {
  return rq_call("rq_dequantize", RQ_DQ, stream, nullptr, odtype, 0, codes, nullptr, ldc, norms, nullptr, n, d,
                 rotors, centroids, bits, xhat, odtype, ldo);
}

kvrq_status rq_quantize_dequantize(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d, int64_t ldx,
                                   const float* rotors, const float* centroids, int bits, uint32_t* codes,
                                   int64_t ldc, float* norms, void* xhat, int64_t ldo) {
  return rq_call("rq_quantize_dequantize", RQ_QDQ, stream, x, xdtype, ldx, nullptr, codes, ldc, nullptr, norms, n, d,
                 rotors, centroids, bits, xhat, xdtype, ldo);
}

// ------------------------------------------------------------------ host-buffer roundtrip
// Device bytes of one chunk slot: x and x_hat rows padded to 16 bytes, code words, norms.
static size_t host_slot_bytes(int d, int bits, kvrq_dtype dt, int64_t rows) {
  const size_t es = dtype_size(dt);
  const size_t row = ((size_t)d * es + 15) / 16 * 16;
  const size_t W = (size_t)kvrq_packed_words(3 * (int64_t)((d + 2) / 3), bits);
  const size_t bytes = (size_t)rows * (2 * row + 4 * W + 4) + 4 * 256;
  return (bytes + 255) / 256 * 256;
}

static kvrq_status pipe_init(DeviceInfo* di) {
  if (di->pipe_ready) return KVRQ_OK;
  cudaError_t e;
  for (int i = 0; i < 3; ++i)
    if ((e = cudaStreamCreateWithFlags(&di->pipe[i], cudaStreamNonBlocking)) != cudaSuccess)
      return cuda_fail("cudaStreamCreateWithFlags", e);
  for (int sl = 0; sl < kHostSlots; ++sl)
    for (cudaEvent_t* ev : {&di->in_done[sl], &di->comp_done[sl], &di->out_done[sl]})
      if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess)
        return cuda_fail("cudaEventCreateWithFlags", e);
  for (cudaEvent_t* ev : {&di->ev_start, &di->ev_end})
    if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess)
      return cuda_fail("cudaEventCreateWithFlags", e);
  di->pipe_ready = true;
  return KVRQ_OK;
}

static kvrq_status copy_rows(void* dst, size_t dpitch, const void* src, size_t spitch, size_t width, int64_t rows,
                             cudaMemcpyKind kind, cudaStream_t st) {
  cudaError_t e = dpitch == width && spitch == width
                      ? cudaMemcpyAsync(dst, src, width * (size_t)rows, kind, st)
                      : cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, (size_t)rows, kind, st);
  return e == cudaSuccess ? KVRQ_OK : cuda_fail("cudaMemcpyAsync", e);
}

static kvrq_status ev_chain(cudaEvent_t ev, cudaStream_t from, cudaStream_t to) {
  cudaError_t e = cudaEventRecord(ev, from);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(to, ev, 0);
  return e == cudaSuccess ? KVRQ_OK : cuda_fail("cudaEventRecord / cudaStreamWaitEvent", e);
}

static kvrq_status rq_host_pipeline(DeviceInfo* di, cudaStream_t caller, const uint8_t* x, kvrq_dtype dt,
                                    int64_t n, int d, int64_t ldx, const float* rotors, const float* centroids,
                                    int bits, uint32_t* codes, int64_t ldc, float* norms, uint8_t* xhat,
                                    int64_t ldo, uint8_t* ws, int64_t chunk) {
  const size_t es = dtype_size(dt);
  const int64_t ld_dev = (int64_t)(((size_t)d * es + 15) / 16 * 16 / es);
  const int64_t W = kvrq_packed_words(3 * (int64_t)((d + 2) / 3), bits);
  const size_t slot = host_slot_bytes(d, bits, dt, chunk);
  cudaStream_t in = di->pipe[0], comp = di->pipe[1], out = di->pipe[2];
  kvrq_status st;
  // everything queued on the caller's stream before this call comes first, and so do the copy-outs
  // of earlier calls (the workspace slots may be the same memory)
  for (cudaStream_t s2 : {in, comp, out})
    if ((st = ev_chain(di->ev_start, caller, s2)) != KVRQ_OK) return st;
  if ((st = ev_chain(di->ev_end, out, in)) != KVRQ_OK) return st;
  for (int64_t r0 = 0, k = 0; r0 < n; r0 += chunk, ++k) {
    const int sl = (int)(k % kHostSlots);
    const int64_t rows = n - r0 < chunk ? n - r0 : chunk;
    uint8_t* b = ws + (size_t)sl * slot;
    uint8_t* dx = b;
    uint8_t* dxh = dx + (size_t)chunk * ld_dev * es;
    uint32_t* dc = reinterpret_cast<uint32_t*>(dxh + (size_t)chunk * ld_dev * es);
    float* dn = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(dc) + ((size_t)chunk * W * 4 + 255) / 256 * 256);
    cudaError_t e;
    if (k >= kHostSlots && (e = cudaStreamWaitEvent(in, di->out_done[sl], 0)) != cudaSuccess)
      return cuda_fail("cudaStreamWaitEvent", e);  // the slot's last copy-out has finished
    if ((st = copy_rows(dx, ld_dev * es, x + (size_t)r0 * ldx * es, ldx * es, d * es, rows, cudaMemcpyHostToDevice,
                        in)) != KVRQ_OK)
      return st;
    if ((st = ev_chain(di->in_done[sl], in, comp)) != KVRQ_OK) return st;
    if ((st = rq_quantize_dequantize(comp, dx, dt, rows, d, ld_dev, rotors, centroids, bits, codes ? dc : nullptr, W,
                                     norms ? dn : nullptr, dxh, ld_dev)) != KVRQ_OK)
      return st;
    if ((st = ev_chain(di->comp_done[sl], comp, out)) != KVRQ_OK) return st;
    if (codes && (st = copy_rows(codes + r0 * ldc, ldc * 4, dc, W * 4, W * 4, rows, cudaMemcpyDeviceToHost, out)) !=
                     KVRQ_OK)
      return st;
    if (norms && (st = copy_rows(norms + r0, 4 * rows, dn, 4 * rows, 4 * rows, 1, cudaMemcpyDeviceToHost, out)) !=
                     KVRQ_OK)
      return st;
    if ((st = copy_rows(xhat + (size_t)r0 * ldo * es, ldo * es, dxh, ld_dev * es, d * es, rows,
                        cudaMemcpyDeviceToHost, out)) != KVRQ_OK)
      return st;
    if ((e = cudaEventRecord(di->out_done[sl], out)) != cudaSuccess) return cuda_fail("cudaEventRecord", e);
  }
  // work queued on the caller's stream after this call waits for the last copy-out
  return ev_chain(di->ev_end, out, caller);
}

size_t kvrq_host_workspace_bytes(int d, int bits, kvrq_dtype dtype, int64_t chunk_rows) {
  if (d < 2 || bits < 1 || bits > 4 || !valid_dtype(dtype) || chunk_rows < 32) return 0;
  return kHostSlots * host_slot_bytes(d, bits, dtype, (chunk_rows + 31) / 32 * 32);
}

kvrq_status rq_quantize_dequantize_host(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d, int64_t ldx,
                                        const float* rotors, const float* centroids, int bits, uint32_t* codes,
                                        int64_t ldc, float* norms, void* xhat, int64_t ldo, void* workspace,
                                        size_t workspace_bytes) {
  const char* name = "rq_quantize_dequantize_host";
  if (n < 0) return set_errorf(KVRQ_EINVAL, "%s: n < 0", name);
  if (d < 2 || d > (1 << 20)) return set_errorf(KVRQ_EINVAL, "%s: d must be in 2..2^20", name);
  if (bits < 1 || bits > 4) return set_errorf(KVRQ_EUNSUPPORTED, "%s: bits must be in 1..4", name);
  if (!valid_dtype(xdtype)) return set_errorf(KVRQ_EINVAL, "%s: bad dtype", name);
  if (n == 0) return KVRQ_OK;
  if (!x || ldx < d || !xhat || ldo < d) return set_errorf(KVRQ_EINVAL, "%s: x, xhat NULL or ldx, ldo < d", name);
  if (codes && ldc < kvrq_packed_words(3 * (int64_t)((d + 2) / 3), bits))
    return set_errorf(KVRQ_EINVAL, "%s: ldc < the code words of a row", name);
  if (!workspace || !aligned(workspace, 256)) return set_errorf(KVRQ_EINVAL, "%s: workspace NULL or not 256-byte aligned", name);
  // the largest chunk of 32-row multiples whose slots fit (at most the whole input)
  int64_t chunk = 32;
  if (kHostSlots * host_slot_bytes(d, bits, xdtype, chunk) > workspace_bytes)
    return set_errorf(KVRQ_EINVAL, "%s: workspace below kvrq_host_workspace_bytes(d, bits, dtype, 32)", name);
  const int64_t cap = (n + 31) / 32 * 32;
  while (chunk * 2 <= cap && kHostSlots * host_slot_bytes(d, bits, xdtype, chunk * 2) <= workspace_bytes) chunk *= 2;
  DeviceInfo* di;
  kvrq_status st = current_device(&di);
  if (st != KVRQ_OK) return st;
  std::lock_guard<std::mutex> lk(di->pipe_mu);
  if ((st = pipe_init(di)) != KVRQ_OK) return st;
  return rq_host_pipeline(di, static_cast<cudaStream_t>(stream), static_cast<const uint8_t*>(x), xdtype, n, d, ldx,
                          rotors, centroids, bits, codes, ldc, norms, static_cast<uint8_t*>(xhat), ldo,
                          static_cast<uint8_t*>(workspace), chunk);
}

kvrq_status pq_quantize_dequantize(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d, int64_t ldx,
                                   const void* pi, const float* centroids, uint32_t* codes, int64_t ldc, void* xhat,
                                   int64_t ldo) {
  return pq_call("pq_quantize_dequantize", PQ_QDQ, stream, x, xdtype, ldx, n, d, pi, centroids, codes, nullptr, ldc,
                 xhat, ldo);
}

kvrq_status pq_dequantize(void* stream, const uint32_t* codes, int64_t ldc, int64_t n, int d, const void* pi,
                          const float* centroids, void* xhat, kvrq_dtype odtype, int64_t ldo) {
  return pq_call("pq_dequantize", PQ_DQ, stream, nullptr, odtype, 0, n, d, pi, centroids, nullptr, codes, ldc, xhat,
                 ldo);
}

kvrq_status rq4_quantize(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d, int64_t ldx,
                         const float* rotors, const float* centroids, int bits, uint32_t* codes, int64_t ldc,
                         float* norms) {
  return rq_call("rq4_quantize", RQ_Q, stream, x, xdtype, ldx, nullptr, codes, ldc, nullptr, norms, n, d, rotors,
                 centroids, bits, nullptr, xdtype, 0, 1, 4);
}

kvrq_status rq4_dequantize(void* stream, const uint32_t* codes, int64_t ldc, const float* norms, int64_t n, int d,
                           const float* rotors, const float* centroids, int bits, void* xhat, kvrq_dtype odtype,
                           int64_t ldo) {
  return rq_call("rq4_dequantize", RQ_DQ, stream, nullptr, odtype, 0, codes, nullptr, ldc, norms, nullptr, n, d,
                 rotors, centroids, bits, xhat, odtype, ldo, 1, 4);
}

kvrq_status rq4_quantize_dequantize(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d, int64_t ldx,
                                    const float* rotors, const float* centroids, int bits, uint32_t* codes,
                                    int64_t ldc, float* norms, void* xhat, int64_t ldo) {
  return rq_call("rq4_quantize_dequantize", RQ_QDQ, stream, x, xdtype, ldx, nullptr, codes, ldc, nullptr, norms, n,
                 d, rotors, centroids, bits, xhat, xdtype, ldo, 1, 4);
}

kvrq_status tq_quantize_mse(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d, int64_t ldx,
                            const void* pi, const float* centroids, int bits, uint32_t* codes, int64_t ldc,
                            float* norms) {
  return tq_call("tq_quantize_mse", TQ_MSE_Q, stream, x, xdtype, ldx, n, d, d, pi, nullptr, centroids, bits, codes,
                 nullptr, ldc, nullptr, nullptr, 0, nullptr, nullptr, norms, nullptr, nullptr, 0);
}

kvrq_status tq_quantize_dequantize_mse(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d, int64_t ldx,
                                       const void* pi, const float* centroids, int bits, uint32_t* codes,
                                       int64_t ldc, float* norms, void* xhat, int64_t ldo) {
  return tq_call("tq_quantize_dequantize_mse", TQ_MSE_QDQ, stream, x, xdtype, ldx, n, d, d, pi, nullptr, centroids,
                 bits, codes, nullptr, ldc, nullptr, nullptr, 0, nullptr, nullptr, norms, nullptr, xhat, ldo);
}

kvrq_status tq_quantize_prod(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d, int64_t ldx,
                             const void* pi, const uint16_t* T, int m, const float* centroids, int bits,
                             uint32_t* codes, int64_t ldc, uint32_t* signs, int64_t lds, float* gammas,
                             float* norms, void* workspace, size_t workspace_bytes) {
  return tq_call("tq_quantize_prod", TQ_PROD_Q, stream, x, xdtype, ldx, n, d, m, pi, T, centroids, bits, codes,
                 nullptr, ldc, signs, nullptr, lds, gammas, nullptr, norms, nullptr, nullptr, 0, 1, workspace,
                 workspace_bytes);
}

kvrq_status tq_dequantize(void* stream, const uint32_t* codes, int64_t ldc, const uint32_t* signs, int64_t lds,
                          const float* gammas, const float* norms, int64_t n, int d, int m, int bits,
                          const void* pi, const uint16_t* T, const float* centroids, void* xhat, kvrq_dtype odtype,
                          int64_t ldo, void* workspace, size_t workspace_bytes) {
  const int mode = signs ? TQ_DQ_PROD : TQ_DQ_MSE;
  return tq_call("tq_dequantize", mode, stream, nullptr, odtype, 0, n, d, m, pi, T, centroids, bits, nullptr, codes,
                 ldc, nullptr, signs, lds, nullptr, gammas, nullptr, norms, xhat, ldo, 1, workspace, workspace_bytes);
}

kvrq_status tq_quantize_prod_noalloc(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d, int64_t ldx,
                                     const void* pi, const uint16_t* T, int m, const float* centroids, int bits,
                                     uint32_t* codes, int64_t ldc, uint32_t* signs, int64_t lds, float* gammas,
                                     float* norms) {
  return tq_call("tq_quantize_prod_noalloc", TQ_PROD_Q, stream, x, xdtype, ldx, n, d, m, pi, T, centroids, bits,
                 codes, nullptr, ldc, signs, nullptr, lds, gammas, nullptr, norms, nullptr, nullptr, 0, 1, nullptr, 0,
                 true);
}

size_t kvrq_tq_workspace_bytes(int64_t rows, int d) {
  if (rows <= 0 || d <= 0) return 0;
  return (size_t)rows * tq_ws_row_bytes(d);
}

kvrq_status qjl_sketch(void* stream, const void* r, kvrq_dtype rdtype, int64_t n, int d, int64_t ldr, const void* T,
                       int m, uint32_t* signs, int64_t lds, float* gammas, int64_t ldn) {
  return qjl_call(stream, r, rdtype, n, d, ldr, T, m, signs, lds, gammas, ldn);
}

}  // extern "C"

// Checks of a paged-cache descriptor shared by the paged calls (tables on the device are not read).
static kvrq_status check_paged(const char* name, const kvrq_paged* pg, int64_t n_heads, int64_t max_tokens) {
  if (!pg->block_tables || !pg->seq_lens || !aligned(pg->block_tables, 4) || !aligned(pg->seq_lens, 4))
    return set_errorf(KVRQ_EINVAL, "%s: block_tables and seq_lens are required", name);
  if (pg->page_tokens < 1 || pg->n_seqs < 1 || pg->kv_heads < 1)
    return set_errorf(KVRQ_EINVAL, "%s: page_tokens, n_seqs and kv_heads must be >= 1", name);
  if (n_heads % ((int64_t)pg->n_seqs * pg->kv_heads) != 0)
    return set_errorf(KVRQ_EINVAL, "%s: n_heads must be a multiple of n_seqs x kv_heads", name);
  if (pg->ld_table < (max_tokens + pg->page_tokens - 1) / pg->page_tokens)
    return set_errorf(KVRQ_EINVAL, "%s: ld_table holds fewer pages than max_tokens needs", name);
  return KVRQ_OK;
}

static kvrq_status score_call(const char* name, void* stream, kvrq_method method, const void* q, kvrq_dtype qdtype,
                              int64_t ldq, int64_t n_heads, int group, int d, int bits, int m, const uint32_t* codes,
                              int64_t ldc, int64_t codes_head_stride, const uint32_t* signs, int64_t lds,
                              int64_t signs_head_stride, const float* norms, const float* gammas,
                              int64_t tok_head_stride, int64_t n_tokens, const kvrq_paged* pg, const float* rotors,
                              const void* pi, kvrq_dtype pi_dtype, const uint16_t* T, const float* centroids,
                              float* scores, int64_t ld_scores) {
  const bool prod = method == KVRQ_TQ_PROD;
  if (method != KVRQ_RQ_MSE && method != KVRQ_TQ_MSE && method != KVRQ_TQ_PROD)
    return set_error(KVRQ_EINVAL, "kv_score_packed: unknown method");
  if (n_heads < 0 || n_tokens < 0 || group < 1) return set_error(KVRQ_EINVAL, "kv_score_packed: bad sizes");
  if (d != 128) return set_error(KVRQ_EUNSUPPORTED, "kv_score_packed: d = 128 is supported");
  if (prod && m != d) return set_error(KVRQ_EUNSUPPORTED, "kv_score_packed: the QJL projection needs m = d");
  const int cbits = prod ? bits - 1 : bits;
  if (cbits < 1 || cbits > 4) return set_error(KVRQ_EUNSUPPORTED, "kv_score_packed: stored code width must be 1..4");
  const int rows_needed = group * (prod ? 2 : 1);
  if (rows_needed > 64) return set_error(KVRQ_EUNSUPPORTED, "kv_score_packed: group too large (<= 64, prod <= 32)");
  if (!valid_dtype(qdtype) || ldq < d) return set_error(KVRQ_EINVAL, "kv_score_packed: bad query dtype or ldq");
  const int ncode = method == KVRQ_RQ_MSE ? 3 * ((d + 2) / 3) : d;
  const int64_t W = kvrq_packed_words(ncode, cbits);
  if (n_heads == 0 || n_tokens == 0) return KVRQ_OK;
  if (!q || !codes || !norms || !centroids || !scores) return set_error(KVRQ_EINVAL, "kv_score_packed: NULL argument");
  // (a paged pool's rows are named by the tables: its strides are the caller's)
  if (ldc < W || ld_scores < n_tokens ||
      (!pg && (tok_head_stride < n_tokens || codes_head_stride < n_tokens * ldc)))
    return set_error(KVRQ_EINVAL, "kv_score_packed: strides too small");
  if (method == KVRQ_RQ_MSE && (!rotors || !aligned(rotors, 16)))
    return set_error(KVRQ_EINVAL, "kv_score_packed: rotors (16-byte aligned) required");
  if (method != KVRQ_RQ_MSE && (!pi || (pi_dtype != KVRQ_F16 && pi_dtype != KVRQ_BF16)))
    return set_error(KVRQ_EINVAL, "kv_score_packed: pi (fp16 or bf16) required");
  if (prod && (!signs || !gammas || !T || lds < m / 32 || (!pg && signs_head_stride < n_tokens * lds)))
    return set_error(KVRQ_EINVAL, "kv_score_packed: signs, gammas and T required for prod");
  if (!aligned(codes, 4) || !aligned(norms, 4) || !aligned(scores, 4))
    return set_error(KVRQ_EINVAL, "kv_score_packed: misaligned pointer");
  if (n_heads > 65535) return set_error(KVRQ_EUNSUPPORTED, "kv_score_packed: more than 65535 heads");
  kvrq_status pst;
  if (pg && (pst = check_paged(name, pg, n_heads, n_tokens)) != KVRQ_OK) return pst;

  DeviceInfo* di;
  kvrq_status st = current_device(&di);
  if (st != KVRQ_OK) return st;
  ScoreArgs a{};
  a.n_heads = n_heads;
  a.group = group;
  a.n_tokens = n_tokens;
  // One CTA runs per SM. A head's tokens are cut into c ranges so that the waves
  // of CTAs times the tiles per CTA (plus the query-rotation prologue, worth about
  // four tiles) is smallest.
  const int64_t tiles = (n_tokens + 127) / 128;
  int64_t best_c = 1, best_cost = -1;
  for (int64_t c = 1; c <= tiles && c <= 256; ++c) {
    const int64_t waves = (n_heads * c + di->num_sms - 1) / di->num_sms;
    const int64_t cost = waves * ((tiles + c - 1) / c + 4);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_c = c;
    }
  }
  a.tokens_per_cta = ((tiles + best_c - 1) / best_c) * 128;
  a.q = q;
  a.ldq = ldq;
  a.q_f32 = qdtype == KVRQ_F32;
  a.q_bf16 = qdtype == KVRQ_BF16;
  a.codes = codes;
  a.ldc = ldc;
  a.codes_head_stride = codes_head_stride;
  a.signs = signs;
  a.lds = lds;
  a.signs_head_stride = signs_head_stride;
  a.norms = norms;
  a.gammas = gammas;
  a.tok_head_stride = tok_head_stride;
  a.rotors = rotors;
  a.pi = pi;
  a.pi_bf16 = pi_dtype == KVRQ_BF16;
  a.T = T;
  a.centroids = centroids;
  a.qjl_scale = (float)(1.2533141373155003 / (double)(prod ? m : d));
  a.scores = scores;
  a.ld_scores = ld_scores;
  a.status = di->status;
  if (pg) {
    a.block_tables = pg->block_tables;
    a.ld_table = pg->ld_table;
    a.seq_lens = pg->seq_lens;
    a.page_tokens = pg->page_tokens;
    a.n_seqs = pg->n_seqs;
    a.kv_heads = pg->kv_heads;
  }
  a.spin_limit = g_wait_limit.load();
  const int nb = rows_needed <= 16 ? 16 : (rows_needed <= 32 ? 32 : 64);
  return launch_status(name, launch_score(method, nb, cbits, a, static_cast<cudaStream_t>(stream)));
}

extern "C" {

kvrq_status kv_score_packed(void* stream, kvrq_method method, const void* q, kvrq_dtype qdtype, int64_t ldq,
                            int64_t n_heads, int group, int d, int bits, int m, const uint32_t* codes, int64_t ldc,
                            int64_t codes_head_stride, const uint32_t* signs, int64_t lds, int64_t signs_head_stride,
                            const float* norms, const float* gammas, int64_t tok_head_stride, int64_t n_tokens,
                            const float* rotors, const void* pi, kvrq_dtype pi_dtype, const uint16_t* T,
                            const float* centroids, float* scores, int64_t ld_scores) {
  return score_call("kv_score_packed", stream, method, q, qdtype, ldq, n_heads, group, d, bits, m, codes, ldc,
                    codes_head_stride, signs, lds, signs_head_stride, norms, gammas, tok_head_stride, n_tokens,
                    nullptr, rotors, pi, pi_dtype, T, centroids, scores, ld_scores);
}

kvrq_status kv_score_packed_paged(void* stream, kvrq_method method, const void* q, kvrq_dtype qdtype, int64_t ldq,
                                  int64_t n_heads, int group, int d, int bits, int m, const uint32_t* codes,
                                  int64_t ldc, int64_t codes_pool_stride, const uint32_t* signs, int64_t lds,
                                  int64_t signs_pool_stride, const float* norms, const float* gammas,
                                  int64_t tok_pool_stride, const kvrq_paged* paged, int64_t max_tokens,
                                  const float* rotors, const void* pi, kvrq_dtype pi_dtype, const uint16_t* T,
                                  const float* centroids, float* scores, int64_t ld_scores) {
  if (!paged) return set_error(KVRQ_EINVAL, "kv_score_packed_paged: paged is NULL");
  return score_call("kv_score_packed_paged", stream, method, q, qdtype, ldq, n_heads, group, d, bits, m, codes, ldc,
                    codes_pool_stride, signs, lds, signs_pool_stride, norms, gammas, tok_pool_stride, max_tokens,
                    paged, rotors, pi, pi_dtype, T, centroids, scores, ld_scores);
}

size_t kvrq_attention_workspace_bytes(int64_t n_heads, int group, int64_t n_tokens) {
  if (n_heads <= 0 || group <= 0 || n_tokens <= 0) return 0;
  return attn_workspace_bytes(n_heads, group, n_tokens);
}

}  // extern "C"

static kvrq_status attention_call(const char* name, void* stream, kvrq_method k_method, const void* q,
                                  kvrq_dtype qdtype, int64_t ldq, int64_t n_heads, int group, int d, float scale,
                                  int k_bits, int m, const uint32_t* k_codes, int64_t ldk, int64_t k_head_stride,
                                  const uint32_t* k_signs, int64_t lds, int64_t s_head_stride, const float* k_norms,
                                  const float* k_gammas, const float* k_rotors, const void* pi, kvrq_dtype pi_dtype,
                                  const uint16_t* T, const float* k_centroids, const uint32_t* v_codes, int64_t ldv,
                                  int64_t v_head_stride, const float* v_norms, int v_bits, const float* v_rotors,
                                  const float* v_centroids, int64_t tok_head_stride, int64_t n_tokens,
                                  const kvrq_paged* pg, void* out, kvrq_dtype odtype, int64_t ldo, void* workspace,
                                  size_t workspace_bytes) {
  const bool prod = k_method == KVRQ_TQ_PROD;
  if (k_method != KVRQ_RQ_MSE && k_method != KVRQ_TQ_MSE && !prod)
    return set_error(KVRQ_EINVAL, "kv_attention_packed: unknown key method");
  if (n_heads < 0 || n_tokens < 0 || group < 1) return set_error(KVRQ_EINVAL, "kv_attention_packed: bad sizes");
  if (d != 128) return set_error(KVRQ_EUNSUPPORTED, "kv_attention_packed: d = 128 is supported");
  if (group > 16) return set_error(KVRQ_EUNSUPPORTED, "kv_attention_packed: group must be <= 16");
  if (prod && m != d) return set_error(KVRQ_EUNSUPPORTED, "kv_attention_packed: the QJL projection needs m = d");
  const int kcb = prod ? k_bits - 1 : k_bits;
  if (kcb < 1 || kcb > 4) return set_error(KVRQ_EUNSUPPORTED, "kv_attention_packed: stored key code width must be 1..4");
  if (v_bits < 1 || v_bits > 4) return set_error(KVRQ_EUNSUPPORTED, "kv_attention_packed: v_bits must be 1..4");
  if (!valid_dtype(qdtype) || ldq < d) return set_error(KVRQ_EINVAL, "kv_attention_packed: bad query dtype or ldq");
  if (!valid_dtype(odtype) || ldo < d) return set_error(KVRQ_EINVAL, "kv_attention_packed: bad output dtype or ldo");
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f)
    return set_error(KVRQ_EINVAL, "kv_attention_packed: scale must be finite");
  if (n_heads == 0) return KVRQ_OK;
  if (n_tokens == 0) return set_error(KVRQ_EINVAL, "kv_attention_packed: no tokens (the softmax is undefined)");
  if (n_heads > 65535) return set_error(KVRQ_EUNSUPPORTED, "kv_attention_packed: more than 65535 heads");
  const int nck = k_method == KVRQ_RQ_MSE ? 3 * ((d + 2) / 3) : d;
  const int64_t Wk = kvrq_packed_words(nck, kcb);
  const int64_t Wv = kvrq_packed_words(3 * ((d + 2) / 3), v_bits);
  if (!q || !k_codes || !k_norms || !k_centroids || !v_codes || !v_norms || !v_rotors || !v_centroids || !out)
    return set_error(KVRQ_EINVAL, "kv_attention_packed: NULL argument");
  if (ldk < Wk || ldv < Wv ||
      (!pg && (k_head_stride < n_tokens * ldk || v_head_stride < n_tokens * ldv || tok_head_stride < n_tokens)))
    return set_error(KVRQ_EINVAL, "kv_attention_packed: strides too small");
  if (k_method == KVRQ_RQ_MSE && (!k_rotors || !aligned(k_rotors, 16)))
    return set_error(KVRQ_EINVAL, "kv_attention_packed: key rotors (16-byte aligned) required");
  if (k_method != KVRQ_RQ_MSE && (!pi || (pi_dtype != KVRQ_F16 && pi_dtype != KVRQ_BF16) || !aligned(pi, 2)))
    return set_error(KVRQ_EINVAL, "kv_attention_packed: pi (fp16 or bf16) required");
  if (prod && (!k_signs || !k_gammas || !T || !aligned(T, 2) || lds < m / 32 ||
               (!pg && s_head_stride < n_tokens * lds)))
    return set_error(KVRQ_EINVAL, "kv_attention_packed: signs, gammas and T required for prod");
  if (!aligned(v_rotors, 16)) return set_error(KVRQ_EINVAL, "kv_attention_packed: value rotors must be 16-byte aligned");
  if (!aligned(k_codes, 4) || !aligned(v_codes, 4) || !aligned(k_norms, 4) || !aligned(v_norms, 4) ||
      (prod && (!aligned(k_signs, 4) || !aligned(k_gammas, 4))) || !aligned(k_centroids, 4) ||
      !aligned(v_centroids, 4) || !aligned(q, qdtype == KVRQ_F32 ? 4 : 2) || !aligned(out, odtype == KVRQ_F32 ? 4 : 2))
    return set_error(KVRQ_EINVAL, "kv_attention_packed: misaligned pointer");
  if (pg) {
    kvrq_status pst = check_paged(name, pg, n_heads, n_tokens);
    if (pst != KVRQ_OK) return pst;
    if (!attn_tc_supported(k_method, kcb, v_bits, group))
      return set_errorf(KVRQ_EUNSUPPORTED, "%s: a paged cache is read by the tensor-core kernel only "
                                           "(kvrq_attention_uses_tensor_cores)", name);
  }
  const size_t need = attn_workspace_bytes(n_heads, group, n_tokens);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 16))
    return set_errorf(KVRQ_EINVAL, "kv_attention_packed: workspace of %zu bytes (16-byte aligned) required", need);

  AttnArgs a{};
  a.n_heads = n_heads;
  a.group = group;
  a.n_tokens = n_tokens;
  a.q = q;
  a.ldq = ldq;
  a.q_f32 = qdtype == KVRQ_F32;
  a.q_bf16 = qdtype == KVRQ_BF16;
  a.scale = scale;
  a.k_codes = k_codes;
  a.ldk = ldk;
  a.k_head_stride = k_head_stride;
  a.k_signs = k_signs;
  a.lds = lds;
  a.s_head_stride = s_head_stride;
  a.k_norms = k_norms;
  a.k_gammas = k_gammas;
  a.k_rotors = k_rotors;
  a.pi = pi;
  a.pi_bf16 = pi_dtype == KVRQ_BF16;
  a.T = T;
  a.k_centroids = k_centroids;
  a.qjl_scale = (float)(1.2533141373155003 / (double)(prod ? m : d));
  a.v_codes = v_codes;
  a.ldv = ldv;
  a.v_head_stride = v_head_stride;
  a.v_norms = v_norms;
  a.v_rotors = v_rotors;
  a.v_centroids = v_centroids;
  a.v_bits = v_bits;
  a.tok_head_stride = tok_head_stride;
  a.out = out;
  a.ldo = ldo;
  a.odtype = odtype;
  const int64_t rows = n_heads * group;
  float* ws = static_cast<float*>(workspace);
  a.ws_q = ws;
  a.ws_sq = ws + rows * kAttnQS;
  a.ws_acc = a.ws_sq + rows * 128;
  // the chunk count (and so the offset of ws_ml) depends on the path; size both regions for the larger
  const int64_t tpc = attn_tokens_per_cta(n_heads, n_tokens), tpi = attn_tc_tokens_per_item(n_heads, n_tokens);
  const int64_t nc_max = std::max((n_tokens + tpc - 1) / tpc, (n_tokens + tpi - 1) / tpi);
  a.ws_ml = a.ws_acc + rows * nc_max * kAttnAS;
  DeviceInfo* di;
  kvrq_status st = current_device(&di);
  if (st != KVRQ_OK) return st;
  a.status = di->status;
  a.spin_limit = g_wait_limit.load();
  if (pg) {
    a.block_tables = pg->block_tables;
    a.ld_table = pg->ld_table;
    a.seq_lens = pg->seq_lens;
    a.page_tokens = pg->page_tokens;
    a.n_seqs = pg->n_seqs;
    a.kv_heads = pg->kv_heads;
  }
  return launch_status(name, launch_attention(k_method, kcb, a, static_cast<cudaStream_t>(stream), di->num_sms));
}

extern "C" {

kvrq_status kv_attention_packed(void* stream, kvrq_method k_method, const void* q, kvrq_dtype qdtype, int64_t ldq,
                                int64_t n_heads, int group, int d, float scale, int k_bits, int m,
                                const uint32_t* k_codes, int64_t ldk, int64_t k_head_stride, const uint32_t* k_signs,
                                int64_t lds, int64_t s_head_stride, const float* k_norms, const float* k_gammas,
                                const float* k_rotors, const void* pi, kvrq_dtype pi_dtype, const uint16_t* T,
                                const float* k_centroids, const uint32_t* v_codes, int64_t ldv, int64_t v_head_stride,
                                const float* v_norms, int v_bits, const float* v_rotors, const float* v_centroids,
                                int64_t tok_head_stride, int64_t n_tokens, void* out, kvrq_dtype odtype, int64_t ldo,
                                void* workspace, size_t workspace_bytes) {
  return attention_call("kv_attention_packed", stream, k_method, q, qdtype, ldq, n_heads, group, d, scale, k_bits, m,
                        k_codes, ldk, k_head_stride, k_signs, lds, s_head_stride, k_norms, k_gammas, k_rotors, pi,
                        pi_dtype, T, k_centroids, v_codes, ldv, v_head_stride, v_norms, v_bits, v_rotors, v_centroids,
                        tok_head_stride, n_tokens, nullptr, out, odtype, ldo, workspace, workspace_bytes);
}

kvrq_status kv_attention_packed_paged(void* stream, kvrq_method k_method, const void* q, kvrq_dtype qdtype,
                                      int64_t ldq, int64_t n_heads, int group, int d, float scale, int k_bits, int m,
                                      const uint32_t* k_codes, int64_t ldk, int64_t k_pool_stride,
                                      const uint32_t* k_signs, int64_t lds, int64_t s_pool_stride,
                                      const float* k_norms, const float* k_gammas, const float* k_rotors,
                                      const void* pi, kvrq_dtype pi_dtype, const uint16_t* T,
                                      const float* k_centroids, const uint32_t* v_codes, int64_t ldv,
                                      int64_t v_pool_stride, const float* v_norms, int v_bits,
                                      const float* v_rotors, const float* v_centroids, int64_t tok_pool_stride,
                                      const kvrq_paged* paged, int64_t max_tokens, void* out, kvrq_dtype odtype,
                                      int64_t ldo, void* workspace, size_t workspace_bytes) {
  if (!paged) return set_error(KVRQ_EINVAL, "kv_attention_packed_paged: paged is NULL");
  return attention_call("kv_attention_packed_paged", stream, k_method, q, qdtype, ldq, n_heads, group, d, scale,
                        k_bits, m, k_codes, ldk, k_pool_stride, k_signs, lds, s_pool_stride, k_norms, k_gammas,
                        k_rotors, pi, pi_dtype, T, k_centroids, v_codes, ldv, v_pool_stride, v_norms, v_bits,
                        v_rotors, v_centroids, tok_pool_stride, max_tokens, paged, out, odtype, ldo, workspace,
                        workspace_bytes);
}

kvrq_status kv_cache_append_rows(void* stream, kvrq_method method, const void* x, kvrq_dtype xdtype, int64_t n_rows,
                                 int d, int64_t ldx, int bits, const float* rotors, const void* pi, const uint16_t* T,
                                 int m, const float* centroids, const int64_t* dst_rows, uint32_t* codes,
                                 int64_t ldc, uint32_t* signs, int64_t lds, float* norms, float* gammas,
                                 int64_t ldn) {
  const char* name = "kv_cache_append_rows";
  if (n_rows > 0 && (!dst_rows || !aligned(dst_rows, 8)))
    return set_error(KVRQ_EINVAL, "kv_cache_append_rows: dst_rows (8-byte aligned) is required");
  switch (method) {
    case KVRQ_RQ_MSE:
      return rq_call(name, RQ_Q, stream, x, xdtype, ldx, nullptr, codes, ldc, nullptr, norms, n_rows, d, rotors,
                     centroids, bits, nullptr, xdtype, 0, ldn, 3, dst_rows);
    case KVRQ_TQ_MSE:
      return tq_call(name, TQ_MSE_Q, stream, x, xdtype, ldx, n_rows, d, d, pi, nullptr, centroids, bits, codes,
                     nullptr, ldc, nullptr, nullptr, 0, nullptr, nullptr, norms, nullptr, nullptr, 0, ldn, nullptr,
                     0, false, dst_rows);
    case KVRQ_TQ_PROD:
      return tq_call(name, TQ_PROD_Q, stream, x, xdtype, ldx, n_rows, d, m, pi, T, centroids, bits, codes, nullptr,
                     ldc, signs, nullptr, lds, gammas, nullptr, norms, nullptr, nullptr, 0, ldn, nullptr, 0, false,
                     dst_rows);
    default:
      return set_error(KVRQ_EINVAL, "kv_cache_append_rows: unknown method");
  }
}

void kvrq_test_fail_allocations(int count) { g_fail_allocs.store(count > 0 ? count : 0); }

void kvrq_set_wait_limit(int64_t polls) {
  g_wait_limit.store(polls < 0 ? -1 : (int32_t)(polls < INT32_MAX ? polls : INT32_MAX));
}

int kvrq_attention_uses_tensor_cores(kvrq_method k_method, int k_bits, int v_bits, int group) {
  const int kcb = k_method == KVRQ_TQ_PROD ? k_bits - 1 : k_bits;
  return attn_tc_supported((int)k_method, kcb, v_bits, group) ? 1 : 0;
}

kvrq_status kv_cache_append(void* stream, kvrq_method method, const void* x, kvrq_dtype xdtype, int64_t n_rows,
                            int d, int64_t ldx, int bits, const float* rotors, const void* pi, const uint16_t* T, int m,
                            const float* centroids, uint32_t* codes, int64_t codes_row_stride, uint32_t* signs,
                            int64_t signs_row_stride, float* norms, float* gammas, int64_t norm_row_stride) {
  switch (method) {
    case KVRQ_RQ_MSE:
      return rq_call("kv_cache_append", RQ_Q, stream, x, xdtype, ldx, nullptr, codes, codes_row_stride, nullptr, norms,
                     n_rows, d, rotors, centroids, bits, nullptr, xdtype, 0, norm_row_stride);
    case KVRQ_TQ_MSE:
      return tq_call("kv_cache_append", TQ_MSE_Q, stream, x, xdtype, ldx, n_rows, d, d, pi, nullptr, centroids, bits,
                     codes, nullptr, codes_row_stride, nullptr, nullptr, 0, nullptr, nullptr, norms, nullptr, nullptr,
                     0, norm_row_stride);
    case KVRQ_TQ_PROD:
      return tq_call("kv_cache_append", TQ_PROD_Q, stream, x, xdtype, ldx, n_rows, d, m, pi, T, centroids, bits, codes,
                     nullptr, codes_row_stride, signs, nullptr, signs_row_stride, gammas, nullptr, norms, nullptr,
                     nullptr, 0, norm_row_stride);
    default:
      return set_error(KVRQ_EINVAL, "kv_cache_append: unknown method");
  }
}

}  // extern "C"
