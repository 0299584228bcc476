// api.cu -- the extern "C" boundary (include/nvfp4.h): argument checks, size
// queries, workspace layout and the linear-layer sequencing.  No kernel code
// here; every step of the path runs in the kernels of amax.cu, quantize.cu
// and gemm.cu.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/nvfp4.h"
#include "common.cuh"
#include "kernels.h"
#include "linear.h"

namespace {

using nvfp4::launch_amax;

inline int64_t pad128(int64_t v) { return (v + 127) / 128 * 128; }
inline int64_t pad4(int64_t v) { return (v + 3) / 4 * 4; }
inline size_t align256(size_t v) { return (v + 255) / 256 * 256; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

struct DeviceInfo {
  int sms = 0;
  bool ok = false;
};

// Per-device SM count and architecture check, queried once.
nvfp4_status device_info(DeviceInfo* out) {
  static std::mutex mu;
  static DeviceInfo cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return NVFP4_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev].ok) {
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return NVFP4_ERR_CUDA;
    if (major != 10) return NVFP4_ERR_DEVICE;
    cache[dev].sms = sms;
    cache[dev].ok = true;
  }
  *out = cache[dev];
  return NVFP4_OK;
}

// Last CUDA error code behind an NVFP4_ERR_CUDA, per host thread.
thread_local int t_last_cuda_error = 0;

inline nvfp4_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return NVFP4_OK;
  t_last_cuda_error = static_cast<int>(e);
  return NVFP4_ERR_CUDA;
}

nvfp4_status check_tensor(const nvfp4_tensor* t, int64_t rows, int64_t cols) {
  if (!t || !t->data || !t->scales || !t->global_scale) return NVFP4_ERR_INVALID_ARG;
  if (t->rows != rows || t->cols != cols) return NVFP4_ERR_SHAPE;
  if (!aligned16(t->data) || !aligned16(t->scales) || (reinterpret_cast<uintptr_t>(t->global_scale) & 3))
    return NVFP4_ERR_ALIGN;
  return NVFP4_OK;
}

// ---------------------------------------------------------------- workspace
constexpr int kWsTensors = 6;
struct WsLayout {
  int64_t rows[kWsTensors], cols[kWsTensors];
  size_t data[kWsTensors], scales[kWsTensors];
  size_t total;
};
// Scalars at offset 0: amax slots (floats 0..7), decode scales (floats 8..15).
// (kAmaxX, kAmaxXr) and (kAmaxDy, kAmaxDyr) are adjacent: one amax pass fills both.
enum { kAmaxX = 0, kAmaxXr = 1, kAmaxW = 2, kAmaxDy = 3, kAmaxDyr = 4 };

WsLayout ws_layout(int64_t T, int64_t Cin, int64_t Cout) {
  WsLayout L;
  const int64_t r[kWsTensors] = {T, Cout, Cin, Cin, T, Cout};
  const int64_t c[kWsTensors] = {Cin, Cin, Cout, T, Cout, T};
  size_t off = 256;
  for (int i = 0; i < kWsTensors; ++i) {
    L.rows[i] = r[i];
    L.cols[i] = c[i];
    L.data[i] = off;
    off = align256(off + static_cast<size_t>(r[i] * c[i] / 2));
    L.scales[i] = off;
    off = align256(off + static_cast<size_t>(pad128(r[i]) * pad4(c[i] / 16)));
  }
  L.total = off;
  return L;
}

nvfp4_tensor ws_tensor(void* ws, const WsLayout& L, int i) {
  uint8_t* b = static_cast<uint8_t*>(ws);
  nvfp4_tensor t;
  t.data = b + L.data[i];
  t.scales = b + L.scales[i];
  t.global_scale = reinterpret_cast<float*>(b) + 8 + i;
  t.rows = L.rows[i];
  t.cols = L.cols[i];
  return t;
}

// Shape rules of the linear layer: multiples of 64, each below 2^31 (the GEMM
// limit), checked before any size arithmetic so ws_layout never overflows.
bool linear_shape_ok(int64_t T, int64_t Cin, int64_t Cout) {
  const int64_t lim = int64_t(1) << 31;
  return T > 0 && Cin > 0 && Cout > 0 && T < lim && Cin < lim && Cout < lim && T % 64 == 0 && Cin % 64 == 0 &&
         Cout % 64 == 0;
}

nvfp4_status linear_check(int64_t T, int64_t Cin, int64_t Cout, void* ws, size_t ws_bytes) {
  if (!linear_shape_ok(T, Cin, Cout)) return NVFP4_ERR_SHAPE;
  if (!ws || ws_bytes < ws_layout(T, Cin, Cout).total) return NVFP4_ERR_WORKSPACE;
  if (!aligned16(ws)) return NVFP4_ERR_ALIGN;
  return NVFP4_OK;
}

// A second stream of the library's own, one per device, created on first use
// (non-blocking), and two events per host thread and device, for the linear
// layer's independent branches.
nvfp4_status side_stream(int* dev_out, cudaStream_t* out) {
  static std::mutex mu;
  static cudaStream_t streams[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return NVFP4_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!streams[dev]) {
    cudaError_t e = cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking);
    if (e != cudaSuccess) return cuda_status(e);
  }
  *dev_out = dev;
  *out = streams[dev];
  return NVFP4_OK;
}

// Fork: the side stream starts after the work enqueued on main so far.  Join:
// main continues after the work enqueued on the side stream since the fork.
// A stream wait binds to the event's latest record when it is enqueued, so a
// thread can re-record its two events in every call; calls from several host
// threads use different events.
struct Fork {
  cudaStream_t main = nullptr, side = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
};

nvfp4_status fork(cudaStream_t main, Fork* f) {
  thread_local cudaEvent_t events[64][2] = {};
  int dev = 0;
  nvfp4_status st = side_stream(&dev, &f->side);
  if (st != NVFP4_OK) return st;
  cudaError_t e = cudaSuccess;
  for (int i = 0; i < 2 && e == cudaSuccess; ++i)
    if (!events[dev][i]) e = cudaEventCreateWithFlags(&events[dev][i], cudaEventDisableTiming);
  if (e != cudaSuccess) return cuda_status(e);
  f->main = main;
  f->start = events[dev][0];
  f->done = events[dev][1];
  e = cudaEventRecord(f->start, main);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(f->side, f->start, 0);
  if (e != cudaSuccess) f->side = nullptr;      // nothing was forked
  return cuda_status(e);
}

nvfp4_status join(Fork* f) {
  if (!f->side) return NVFP4_OK;
  cudaError_t e = cudaEventRecord(f->done, f->side);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(f->main, f->done, 0);
  f->side = nullptr;
  return cuda_status(e);
}

// After an error on one branch: main still waits for what the side stream
// already holds, so the caller's buffers stay in use until both are done.
nvfp4_status fail(Fork* f, nvfp4_status st) {
  (void)join(f);
  return st;
}

}  // namespace

namespace nvfp4 {

size_t linear_forward_bytes(int64_t T, int64_t Cin, int64_t Cout) {
  if (!linear_shape_ok(T, Cin, Cout)) return 0;
  return ws_layout(T, Cin, Cout).data[3];   // tensors 0..2 and the scalars come first
}

nvfp4_status linear_forward(const void* X, const void* W, int64_t T, int64_t Cin, int64_t Cout, void* Y, void* ws,
                            bool keep_wgrad, nvfp4_stream_t stream) {
  const WsLayout L = ws_layout(T, Cin, Cout);
  float* amax = static_cast<float*>(ws);
  const nvfp4_tensor xr = ws_tensor(ws, L, 0), wr = ws_tensor(ws, L, 1), wc = ws_tensor(ws, L, 2);
  nvfp4_status st;
  // W's amax and 2D copies (RN) on the side stream while X's run on the caller's
  // stream (without the wgrad operand -- the allocation-free forward -- both run
  // on the caller's stream: it creates no stream or event)
  Fork f;
  cudaStream_t wstream = reinterpret_cast<cudaStream_t>(stream);
  if (keep_wgrad) {
    if ((st = fork(wstream, &f)) != NVFP4_OK) return st;
    wstream = f.side;
  }
  nvfp4_stream_t ws_ = reinterpret_cast<nvfp4_stream_t>(wstream);
  if ((st = nvfp4_amax(W, Cout, Cin, Cin, 0, amax + kAmaxW, ws_)) != NVFP4_OK ||
      (st = nvfp4_quantize(W, Cout, Cin, Cin, NVFP4_2D, 0, 0, 0, amax + kAmaxW, &wr, &wc, ws_)) != NVFP4_OK)
    return fail(&f, st);
  // one pass over X gives both its amax (row copy) and its RHT amax (column copy)
  if ((st = nvfp4_amax(X, T, Cin, Cin, 2, amax + kAmaxX, stream)) != NVFP4_OK) return fail(&f, st);
  if (keep_wgrad) {
    // the X row copy (fprop) and the X^T copy with the RHT along tokens, saved
    // for wgrad, from one read of X; amax + kAmaxX holds [max|X|, max|Q X|]
    const nvfp4_tensor xc = ws_tensor(ws, L, 3);
    if ((st = nvfp4_quantize(X, T, Cin, Cin, NVFP4_ROWCOL, 1, 0, 0, amax + kAmaxX, &xr, &xc, stream)) != NVFP4_OK)
      return fail(&f, st);
    if ((st = join(&f)) != NVFP4_OK) return st;
  } else if ((st = nvfp4_quantize(X, T, Cin, Cin, NVFP4_ROW, 0, 0, 0, amax + kAmaxX, &xr, nullptr, stream)) !=
             NVFP4_OK) {
    return st;
  }
  return nvfp4_gemm(&xr, &wr, Y, NVFP4_OUT_BF16, Cout, stream);
}

}  // namespace nvfp4

extern "C" {

size_t nvfp4_data_bytes(int64_t rows, int64_t cols) {
  return (rows > 0 && cols > 0) ? static_cast<size_t>(rows * (cols / 2)) : 0;
}

size_t nvfp4_scale_bytes(int64_t rows, int64_t cols) {
  return (rows > 0 && cols > 0) ? static_cast<size_t>(pad128(rows) * pad4(cols / 16)) : 0;
}

size_t nvfp4_mx_scale_bytes(int64_t rows, int64_t cols) {
  return (rows > 0 && cols > 0) ? static_cast<size_t>(pad128(rows) * pad4(cols / 32)) : 0;
}

nvfp4_status nvfp4_mx_quantize(const void* x, int64_t R, int64_t C, int64_t ld, const nvfp4_tensor* out,
                               nvfp4_stream_t stream) {
  if (!x || !out) return NVFP4_ERR_INVALID_ARG;
  if (R <= 0 || C <= 0 || ld < C || C % 32) return NVFP4_ERR_SHAPE;
  if (!aligned16(x) || ld % 8) return NVFP4_ERR_ALIGN;
  nvfp4_status st;
  if ((st = check_tensor(out, R, C)) != NVFP4_OK) return st;
  DeviceInfo di;
  if ((st = device_info(&di)) != NVFP4_OK) return st;
  return cuda_status(nvfp4::launch_mx_quant_row(x, R, C, ld, out->data, out->scales, out->global_scale, di.sms,
                                                reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_mx_gemm(const nvfp4_tensor* A, const nvfp4_tensor* B, void* D, nvfp4_out_dtype out_dtype,
                           int64_t ldd, nvfp4_stream_t stream) {
  if (!A || !B || !D) return NVFP4_ERR_INVALID_ARG;
  if (out_dtype != NVFP4_OUT_F32 && out_dtype != NVFP4_OUT_BF16) return NVFP4_ERR_INVALID_ARG;
  const int64_t M = A->rows, N = B->rows, K = A->cols;
  if (M <= 0 || N <= 0 || K <= 0 || B->cols != K) return NVFP4_ERR_SHAPE;
  if (K % 32 || N % 16 || ldd < N || M >= (1LL << 31) || N >= (1LL << 31) || K >= (1LL << 31))
    return NVFP4_ERR_SHAPE;
  nvfp4_status st;
  if ((st = check_tensor(A, M, K)) != NVFP4_OK || (st = check_tensor(B, N, K)) != NVFP4_OK) return st;
  if (!aligned16(D) || ldd % 8) return NVFP4_ERR_ALIGN;
  DeviceInfo di;
  if ((st = device_info(&di)) != NVFP4_OK) return st;
  return cuda_status(nvfp4::launch_gemm(A->data, A->scales, A->global_scale, B->data, B->scales, B->global_scale,
                                        M, N, K, D, out_dtype == NVFP4_OUT_BF16, ldd, di.sms,
                                        reinterpret_cast<cudaStream_t>(stream), 1));
}

uint32_t nvfp4_rht_sign_mask(void) { return nvfp4::kRhtSignMask; }

nvfp4_status nvfp4_selftest_scale_division(uint64_t* bad_quotients, uint64_t* bad_codes) {
  if (!bad_quotients || !bad_codes) return NVFP4_ERR_INVALID_ARG;
  DeviceInfo di;
  nvfp4_status st = device_info(&di);
  if (st != NVFP4_OK) return st;
  unsigned long long q = 0, c = 0;
  st = cuda_status(nvfp4::selftest_div6(&q, &c, di.sms));
  *bad_quotients = q;
  *bad_codes = c;
  return st;
}

nvfp4_status nvfp4_selftest_sr_rounding(uint64_t* mismatches, uint64_t* checked) {
  if (!mismatches || !checked) return NVFP4_ERR_INVALID_ARG;
  DeviceInfo di;
  nvfp4_status st = device_info(&di);
  if (st != NVFP4_OK) return st;
  unsigned long long m = 0, c = 0;
  st = cuda_status(nvfp4::selftest_sr(&m, &c));
  *mismatches = m;
  *checked = c;
  return st;
}

int nvfp4_version(void) { return 1; }

int nvfp4_last_cuda_error(const char** name) {
  const int e = t_last_cuda_error;
  if (name) *name = cudaGetErrorName(static_cast<cudaError_t>(e));
  return e;
}

const char* nvfp4_status_string(nvfp4_status s) {
  switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_SHAPE: return "shape breaks a divisibility rule";
    case NVFP4_ERR_ALIGN: return "pointer or pitch misaligned";
    case NVFP4_ERR_UNSUPPORTED: return "mode/flag combination not supported";
    case NVFP4_ERR_DEVICE: return "device is not sm_100";
    case NVFP4_ERR_CUDA: return "CUDA launch or driver call failed";
    case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
    case NVFP4_ERR_TIMEOUT: return "a kernel gave up on a bounded wait";
  }
  return "unknown status";
}

nvfp4_status nvfp4_amax(const void* x, int64_t R, int64_t C, int64_t ld, int rht, float* amax_dev,
                        nvfp4_stream_t stream) {
  if (!x || !amax_dev || rht < 0 || rht > 2) return NVFP4_ERR_INVALID_ARG;
  if (R < 0 || C < 0 || ld < C) return NVFP4_ERR_SHAPE;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(amax_dev) & 3)) return NVFP4_ERR_ALIGN;
  if (rht && (R % 16 || C % 4)) return NVFP4_ERR_SHAPE;
  if (rht && ld % 4) return NVFP4_ERR_ALIGN;
  DeviceInfo di;
  nvfp4_status st = device_info(&di);
  if (st != NVFP4_OK) return st;
  return cuda_status(launch_amax(x, R, C, ld, rht, amax_dev, di.sms,
                                 reinterpret_cast<cudaStream_t>(stream)));
}

static nvfp4_status quantize_checked(const void* x, int64_t R, int64_t C, int64_t ld, nvfp4_mode mode, int rht,
                                     int sr, uint64_t seed, int64_t row0, const float* amax_dev,
                                     const nvfp4_tensor* row_out, const nvfp4_tensor* col_out,
                                     nvfp4_stream_t stream) {
  if (!x || !amax_dev) return NVFP4_ERR_INVALID_ARG;
  if (mode != NVFP4_ROW && mode != NVFP4_COL && mode != NVFP4_ROWCOL && mode != NVFP4_2D)
    return NVFP4_ERR_INVALID_ARG;
  if (R <= 0 || C <= 0 || ld < C) return NVFP4_ERR_SHAPE;
  if (!aligned16(x) || ld % 8) return NVFP4_ERR_ALIGN;
  if (rht && mode != NVFP4_COL && mode != NVFP4_ROWCOL) return NVFP4_ERR_UNSUPPORTED;
  if (sr && mode == NVFP4_2D) return NVFP4_ERR_UNSUPPORTED;
  if (row0 < 0 || row0 % 16 || row0 >= (int64_t(1) << 40)) return NVFP4_ERR_SHAPE;
  if (row0 && row0 + R > (int64_t(1) << 62) / C) return NVFP4_ERR_SHAPE;  // (row0 + R) * C stays in int64
  if (row0 && mode == NVFP4_2D) return NVFP4_ERR_UNSUPPORTED;
  const bool want_row = mode == NVFP4_ROW || mode == NVFP4_ROWCOL || (mode == NVFP4_2D && row_out);
  const bool want_col = mode == NVFP4_COL || mode == NVFP4_ROWCOL || (mode == NVFP4_2D && col_out);
  if (mode == NVFP4_2D && !want_row && !want_col) return NVFP4_ERR_INVALID_ARG;
  if (want_row && C % 16) return NVFP4_ERR_SHAPE;
  if (want_col && (R % 16 || C % 4)) return NVFP4_ERR_SHAPE;
  if (mode == NVFP4_2D && (R % 16 || C % 16)) return NVFP4_ERR_SHAPE;
  nvfp4_status st;
  if (want_row && (st = check_tensor(row_out, R, C)) != NVFP4_OK) return st;
  if (want_col && (st = check_tensor(col_out, C, R)) != NVFP4_OK) return st;
  DeviceInfo di;
  if ((st = device_info(&di)) != NVFP4_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (mode == NVFP4_2D) {
    e = nvfp4::launch_quant_2d(x, R, C, ld, amax_dev, want_row ? row_out->data : nullptr,
                               want_row ? row_out->scales : nullptr, want_row ? row_out->global_scale : nullptr,
                               want_col ? col_out->data : nullptr, want_col ? col_out->scales : nullptr,
                               want_col ? col_out->global_scale : nullptr, di.sms, s);
    return cuda_status(e);
  }
  // ROWCOL with RHT: the row copy takes amax_dev[0], the RHT column copy amax_dev[1]
  const float* amax_col = (mode == NVFP4_ROWCOL && rht) ? amax_dev + 1 : amax_dev;
  if (mode == NVFP4_ROWCOL && !sr) {   // both copies from one read of x
    e = nvfp4::launch_quant_rowcol(x, R, C, ld, amax_dev, amax_col, rht, row_out->data, row_out->scales,
                                   row_out->global_scale, col_out->data, col_out->scales, col_out->global_scale,
                                   di.sms, s);
    return cuda_status(e);
  }
  if (want_row) {
    e = nvfp4::launch_quant_row(x, R, C, ld, amax_dev, sr, seed, row0 * C, row_out->data, row_out->scales,
                                row_out->global_scale, di.sms, s);
    if (e != cudaSuccess) return cuda_status(e);
  }
  if (want_col) {
    e = nvfp4::launch_quant_col(x, R, C, ld, amax_col, rht, sr, seed, row0 * C, col_out->data,
                                col_out->scales, col_out->global_scale, di.sms, s);
    if (e != cudaSuccess) return cuda_status(e);
  }
  return NVFP4_OK;
}

nvfp4_status nvfp4_quantize(const void* x, int64_t R, int64_t C, int64_t ld, nvfp4_mode mode, int rht, int sr,
                            uint64_t seed, const float* amax_dev, const nvfp4_tensor* row_out,
                            const nvfp4_tensor* col_out, nvfp4_stream_t stream) {
  return quantize_checked(x, R, C, ld, mode, rht, sr, seed, 0, amax_dev, row_out, col_out, stream);
}

nvfp4_status nvfp4_quantize_rows(const void* x, int64_t R, int64_t C, int64_t ld, nvfp4_mode mode, int rht,
                                 int sr, uint64_t seed, int64_t row0, const float* amax_dev,
                                 const nvfp4_tensor* row_out, const nvfp4_tensor* col_out, nvfp4_stream_t stream) {
  return quantize_checked(x, R, C, ld, mode, rht, sr, seed, row0, amax_dev, row_out, col_out, stream);
}

static nvfp4_status gemm_checked(const nvfp4_tensor* A, const nvfp4_tensor* B, void* D, nvfp4_out_dtype out_dtype,
                          int64_t ldd, float* amax_out, nvfp4_stream_t stream) {
  if (!A || !B || !D) return NVFP4_ERR_INVALID_ARG;
  if (out_dtype != NVFP4_OUT_F32 && out_dtype != NVFP4_OUT_BF16) return NVFP4_ERR_INVALID_ARG;
  const int64_t M = A->rows, N = B->rows, K = A->cols;
  if (M <= 0 || N <= 0 || K <= 0 || B->cols != K) return NVFP4_ERR_SHAPE;
  if (K % 32 || N % 16 || ldd < N || M >= (1LL << 31) || N >= (1LL << 31) || K >= (1LL << 31))
    return NVFP4_ERR_SHAPE;
  nvfp4_status st;
  if ((st = check_tensor(A, M, K)) != NVFP4_OK || (st = check_tensor(B, N, K)) != NVFP4_OK) return st;
  if (!aligned16(D) || ldd % 8) return NVFP4_ERR_ALIGN;
  DeviceInfo di;
  if ((st = device_info(&di)) != NVFP4_OK) return st;
  return cuda_status(nvfp4::launch_gemm(A->data, A->scales, A->global_scale, B->data, B->scales, B->global_scale,
                                        M, N, K, D, out_dtype == NVFP4_OUT_BF16, ldd, di.sms,
                                        reinterpret_cast<cudaStream_t>(stream), 0, amax_out));
}

nvfp4_status nvfp4_gemm(const nvfp4_tensor* A, const nvfp4_tensor* B, void* D, nvfp4_out_dtype out_dtype,
                        int64_t ldd, nvfp4_stream_t stream) {
  return gemm_checked(A, B, D, out_dtype, ldd, nullptr, stream);
}

nvfp4_status nvfp4_gemm_amax(const nvfp4_tensor* A, const nvfp4_tensor* B, void* D, nvfp4_out_dtype out_dtype,
                             int64_t ldd, float* amax_dev, nvfp4_stream_t stream) {
  if (!amax_dev) return NVFP4_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(amax_dev) % 4) return NVFP4_ERR_ALIGN;
  return gemm_checked(A, B, D, out_dtype, ldd, amax_dev, stream);
}

size_t nvfp4_linear_workspace_bytes(int64_t T, int64_t Cin, int64_t Cout) {
  const int64_t lim = int64_t(1) << 31;
  if (T <= 0 || Cin <= 0 || Cout <= 0 || T >= lim || Cin >= lim || Cout >= lim) return 0;
  return ws_layout(T, Cin, Cout).total;
}

nvfp4_status nvfp4_linear_workspace_tensor(void* workspace, int64_t T, int64_t Cin, int64_t Cout, int which,
                                           nvfp4_tensor* out) {
  if (!workspace || !out || which < 0 || which >= kWsTensors) return NVFP4_ERR_INVALID_ARG;
  const int64_t lim = int64_t(1) << 31;
  if (T <= 0 || Cin <= 0 || Cout <= 0 || T >= lim || Cin >= lim || Cout >= lim) return NVFP4_ERR_SHAPE;
  *out = ws_tensor(workspace, ws_layout(T, Cin, Cout), which);
  return NVFP4_OK;
}

nvfp4_status nvfp4_linear_fwd(const void* X, const void* W, int64_t T, int64_t Cin, int64_t Cout, void* Y,
                              void* workspace, size_t workspace_bytes, nvfp4_stream_t stream) {
  if (!X || !W || !Y) return NVFP4_ERR_INVALID_ARG;
  nvfp4_status st = linear_check(T, Cin, Cout, workspace, workspace_bytes);
  if (st != NVFP4_OK) return st;
  if (!aligned16(X) || !aligned16(W) || !aligned16(Y)) return NVFP4_ERR_ALIGN;
  return nvfp4::linear_forward(X, W, T, Cin, Cout, Y, workspace, true, stream);
}

nvfp4_status nvfp4_linear_bwd(const void* dY, int64_t T, int64_t Cin, int64_t Cout, uint64_t seed, void* dX,
                              float* dW, void* workspace, size_t workspace_bytes, nvfp4_stream_t stream) {
  if (!dY || !dX || !dW) return NVFP4_ERR_INVALID_ARG;
  nvfp4_status st = linear_check(T, Cin, Cout, workspace, workspace_bytes);
  if (st != NVFP4_OK) return st;
  if (!aligned16(dY) || !aligned16(dX) || !aligned16(dW)) return NVFP4_ERR_ALIGN;
  const WsLayout L = ws_layout(T, Cin, Cout);
  float* amax = static_cast<float*>(workspace);
  const nvfp4_tensor wc = ws_tensor(workspace, L, 2), xc = ws_tensor(workspace, L, 3),
                     gr = ws_tensor(workspace, L, 4), gc = ws_tensor(workspace, L, 5);
  // one pass over dY gives both its amax (row copy) and its RHT amax (column copy)
  if ((st = nvfp4_amax(dY, T, Cout, Cout, 2, amax + kAmaxDy, stream)) != NVFP4_OK) return st;
  // wgrad: dW = dY^T X, both with the RHT along tokens, SR on dY
  if ((st = nvfp4_quantize(dY, T, Cout, Cout, NVFP4_COL, 1, 1, seed, amax + kAmaxDyr, nullptr, &gc, stream)) !=
      NVFP4_OK)
    return st;
  // the dY row copy (SR) for dgrad on the side stream, next to the wgrad GEMM:
  // the quantizer is bound by the integer ALU pipe, the GEMM by the tensor pipe,
  // and its CTAs fit beside the GEMM's on every SM
  Fork f;
  if ((st = fork(reinterpret_cast<cudaStream_t>(stream), &f)) != NVFP4_OK) return st;
  if ((st = nvfp4_gemm(&gc, &xc, dW, NVFP4_OUT_F32, Cin, stream)) != NVFP4_OK ||
      (st = nvfp4_quantize(dY, T, Cout, Cout, NVFP4_ROW, 0, 1, seed, amax + kAmaxDy, &gr, nullptr,
                           reinterpret_cast<nvfp4_stream_t>(f.side))) != NVFP4_OK)
    return fail(&f, st);
  if ((st = join(&f)) != NVFP4_OK) return st;
  // dgrad: dX = dY W, dY row-wise with SR, W^T from the 2D column copy
  return nvfp4_gemm(&gr, &wc, dX, NVFP4_OUT_BF16, Cin, stream);
}

nvfp4_status nvfp4_read_device_error(unsigned int* code, int clear) {
  if (!code) return NVFP4_ERR_INVALID_ARG;
  return cuda_status(nvfp4::read_device_error(code, clear));
}

nvfp4_status nvfp4_wait_probe(uint32_t timeout_us, nvfp4_stream_t stream) {
  DeviceInfo di;
  nvfp4_status st = device_info(&di);
  if (st != NVFP4_OK) return st;
  return cuda_status(nvfp4::launch_wait_probe(timeout_us, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
