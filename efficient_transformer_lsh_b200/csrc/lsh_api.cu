// C ABI of the LSH-attention library: argument checks, workspace sizing,
// dispatch to the kernels, and the device status word.
#include <atomic>
#include <initializer_list>
#include <cmath>
#include <mutex>

#include "internal.h"
#include "tc_common.cuh"

namespace lsh {
namespace {

// One thread waits, through the bounded wait of the tensor-core pipelines, on
// a barrier that nothing arrives on; the wait runs out after limit_ns and
// records LSH_ERR_TIMEOUT. No asynchronous copy or MMA is in flight.
__global__ void wait_timeout_kernel(uint64_t limit_ns, int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    abort = 0;
    tc::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) tc::mbar_wait(&bar, 0u, (volatile int*)&abort, status, limit_ns);
}

std::atomic<uint64_t> g_launches{0};

// Device status word: kernels record LSH_ERR_TIMEOUT / LSH_ERR_DEVICE_CHECK
// here instead of trapping, so the context stays usable.
__device__ int g_status_word;

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {};
std::mutex g_status_mu;

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

lsh_status check_problem(const lsh_problem* p) {
  if (!p) return LSH_ERR_INVALID_ARG;
  if (p->B < 0 || p->H < 0 || p->L < 0 || p->d <= 0) return LSH_ERR_INVALID_ARG;
  if (p->n_buckets < 2 || p->n_buckets % 2 != 0 || p->n_buckets > 65536) return LSH_ERR_INVALID_ARG;
  if (p->n_rounds < 1 || p->n_rounds > 64) return LSH_ERR_INVALID_ARG;
  if (p->chunk <= 0) return LSH_ERR_INVALID_ARG;
  if (p->L % p->chunk != 0) return LSH_ERR_INVALID_ARG;
  if (p->causal != 0 && p->causal != 1) return LSH_ERR_INVALID_ARG;
  if (!std::isfinite(p->scale)) return LSH_ERR_INVALID_ARG;
  if (p->dtype != LSH_F32 && p->dtype != LSH_BF16) return LSH_ERR_INVALID_ARG;
  if (p->d != kDHead) return LSH_ERR_UNSUPPORTED;
  if (p->chunk % 64 != 0) return LSH_ERR_UNSUPPORTED;
  // int32 positions, and per-round index spaces addressed in 32 bits
  const int64_t rows = (int64_t)p->B * p->H * p->L;
  if ((int64_t)p->n_rounds * rows > (int64_t)INT32_MAX) return LSH_ERR_UNSUPPORTED;
  if ((int64_t)p->B * p->H * p->n_rounds * (p->L / 64) > (int64_t)INT32_MAX)
    return LSH_ERR_UNSUPPORTED;
  return LSH_OK;
}

bool empty(const lsh_problem* p) { return (int64_t)p->B * p->H * p->L == 0; }

lsh_status cuda_status(cudaError_t e) { return e == cudaSuccess ? LSH_OK : LSH_ERR_CUDA; }

}  // namespace

void note_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

int* device_status_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_status_mu);
  if (!g_status_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_status_word) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = (int*)ptr;
  }
  return g_status_ptr[dev];
}

}  // namespace lsh

using namespace lsh;

extern "C" {

lsh_status lsh_hash(const lsh_problem* p, const void* qk, const void* R, int32_t* bucket,
                    lsh_stream_t stream) {
  lsh_status st = check_problem(p);
  if (st != LSH_OK) return st;
  if (empty(p)) return LSH_OK;
  if (!qk || !R || !bucket) return LSH_ERR_INVALID_ARG;
  if (!aligned(qk, 16)) return LSH_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (p->dtype == LSH_BF16) {
    int* status = device_status_word();
    cudaError_t e = launch_hash_tc(*p, qk, R, bucket, status, s);
    if (e != cudaErrorNotSupported) return cuda_status(e);
  }
  return cuda_status(launch_hash_simt(*p, qk, R, bucket, s));
}

size_t lsh_sort_workspace_size(const lsh_problem* p) {
  if (check_problem(p) != LSH_OK) return 0;
  return sort_ws_bytes(*p);
}

lsh_status lsh_sort(const lsh_problem* p, const int32_t* bucket, int32_t* perm, void* ws,
                    size_t ws_bytes, lsh_stream_t stream) {
  lsh_status st = check_problem(p);
  if (st != LSH_OK) return st;
  if (empty(p)) return LSH_OK;
  if (!bucket || !perm) return LSH_ERR_INVALID_ARG;
  if (!ws || ws_bytes < sort_ws_bytes(*p) || !aligned(ws, 256)) return LSH_ERR_WORKSPACE;
  return cuda_status(launch_sort(*p, bucket, perm, sort_ws_carve(*p, ws), device_status_word(),
                                 (cudaStream_t)stream));
}

size_t lsh_fwd_workspace_size(const lsh_problem* p) {
  if (check_problem(p) != LSH_OK) return 0;
  return fwd_ws_bytes(*p);
}

lsh_status lsh_attn_fwd(const lsh_problem* p, const void* qk, const void* v, const int32_t* perm,
                        void* out, void* out_lo, float* lse, void* ws, size_t ws_bytes,
                        lsh_stream_t stream) {
  lsh_status st = check_problem(p);
  if (st != LSH_OK) return st;
  if (empty(p)) return LSH_OK;
  if (!qk || !v || !perm || !out || !lse) return LSH_ERR_INVALID_ARG;
  if (!aligned(qk, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(out_lo, 16))
    return LSH_ERR_INVALID_ARG;
  if (!ws || ws_bytes < fwd_ws_bytes(*p) || !aligned(ws, 256)) return LSH_ERR_WORKSPACE;
  if (p->dtype == LSH_F32) out_lo = nullptr;
  return cuda_status(launch_attn_fwd(*p, qk, v, perm, out, out_lo, lse, fwd_ws_carve(*p, ws),
                                     device_status_word(), (cudaStream_t)stream));
}

size_t lsh_bwd_workspace_size(const lsh_problem* p) {
  if (check_problem(p) != LSH_OK) return 0;
  return bwd_ws_bytes(*p);
}

lsh_status lsh_attn_bwd(const lsh_problem* p, const void* qk, const void* v, const int32_t* perm,
                        const void* out, const void* out_lo, const float* lse, const void* dout,
                        float* dqk, float* dv, void* ws, size_t ws_bytes, lsh_stream_t stream) {
  lsh_status st = check_problem(p);
  if (st != LSH_OK) return st;
  if (empty(p)) return LSH_OK;
  if (!qk || !v || !perm || !out || !lse || !dout || !dqk || !dv) return LSH_ERR_INVALID_ARG;
  if (!aligned(qk, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(dout, 16) ||
      !aligned(dqk, 16) || !aligned(dv, 16) || !aligned(out_lo, 16))
    return LSH_ERR_INVALID_ARG;
  if (!ws || ws_bytes < bwd_ws_bytes(*p) || !aligned(ws, 256)) return LSH_ERR_WORKSPACE;
  if (p->dtype == LSH_F32) out_lo = nullptr;
  return cuda_status(launch_attn_bwd(*p, qk, v, perm, out, out_lo, lse, dout, dqk, dv, ws,
                                     device_status_word(), (cudaStream_t)stream));
}

static lsh_status check_local(const lsh_problem* p, int32_t n_back, int32_t n_fwd) {
  lsh_status st = check_problem(p);
  if (st != LSH_OK) return st;
  if (p->n_rounds != 1 || n_back < 0 || n_fwd < 0 || n_back > 65536 || n_fwd > 65536)
    return LSH_ERR_INVALID_ARG;
  return LSH_OK;
}

size_t lsh_local_fwd_workspace_size(const lsh_problem* p, int32_t n_back, int32_t n_fwd) {
  if (check_local(p, n_back, n_fwd) != LSH_OK) return 0;
  return local_fwd_ws_bytes(*p, n_back, n_fwd);
}

lsh_status lsh_local_attn_fwd(const lsh_problem* p, int32_t n_back, int32_t n_fwd, const void* qk,
                              const void* v, void* out, void* out_lo, float* lse, void* ws,
                              size_t ws_bytes, lsh_stream_t stream) {
  lsh_status st = check_local(p, n_back, n_fwd);
  if (st != LSH_OK) return st;
  if (empty(p)) return LSH_OK;
  if (!qk || !v || !out || !lse) return LSH_ERR_INVALID_ARG;
  if (!aligned(qk, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(out_lo, 16))
    return LSH_ERR_INVALID_ARG;
  if (!ws || ws_bytes < local_fwd_ws_bytes(*p, n_back, n_fwd) || !aligned(ws, 256))
    return LSH_ERR_WORKSPACE;
  if (p->dtype == LSH_F32) out_lo = nullptr;
  return cuda_status(launch_local_fwd(*p, n_back, n_fwd, qk, v, out, out_lo, lse, ws,
                                      device_status_word(), (cudaStream_t)stream));
}

size_t lsh_local_bwd_workspace_size(const lsh_problem* p, int32_t n_back, int32_t n_fwd) {
  if (check_local(p, n_back, n_fwd) != LSH_OK) return 0;
  return local_bwd_ws_bytes(*p, n_back, n_fwd);
}

lsh_status lsh_local_attn_bwd(const lsh_problem* p, int32_t n_back, int32_t n_fwd, const void* qk,
                              const void* v, const void* out, const void* out_lo, const float* lse,
                              const void* dout, float* dqk, float* dv, void* ws, size_t ws_bytes,
                              lsh_stream_t stream) {
  lsh_status st = check_local(p, n_back, n_fwd);
  if (st != LSH_OK) return st;
  if (empty(p)) return LSH_OK;
  if (!qk || !v || !out || !lse || !dout || !dqk || !dv) return LSH_ERR_INVALID_ARG;
  if (!aligned(qk, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(dout, 16) ||
      !aligned(dqk, 16) || !aligned(dv, 16) || !aligned(out_lo, 16))
    return LSH_ERR_INVALID_ARG;
  if (!ws || ws_bytes < local_bwd_ws_bytes(*p, n_back, n_fwd) || !aligned(ws, 256))
    return LSH_ERR_WORKSPACE;
  if (p->dtype == LSH_F32) out_lo = nullptr;
  return cuda_status(launch_local_bwd(*p, n_back, n_fwd, qk, v, out, out_lo, lse, dout, dqk, dv,
                                      ws, device_status_word(), (cudaStream_t)stream));
}

static lsh_status check_ff(const lsh_ff_problem* f) {
  if (!f) return LSH_ERR_INVALID_ARG;
  if (f->B < 0 || f->H < 1 || f->L < 0 || f->d_ff < 128 || f->ff_chunk < 128)
    return LSH_ERR_INVALID_ARG;
  if (f->L % 128 != 0 || f->d_ff % 128 != 0 || f->ff_chunk % 128 != 0) return LSH_ERR_INVALID_ARG;
  if (f->d_ff > 65536 || 64 * (int64_t)f->H > 65536) return LSH_ERR_UNSUPPORTED;
  if ((int64_t)f->B * f->H * f->L * 64 > (int64_t)INT32_MAX * 64 ||
      (int64_t)f->B * f->L > (int64_t)INT32_MAX / 2)
    return LSH_ERR_UNSUPPORTED;
  return LSH_OK;
}
static bool ff_empty(const lsh_ff_problem* f) { return (int64_t)f->B * f->L == 0; }
static bool all_aligned16(std::initializer_list<const void*> ps) {
  for (const void* q : ps)
    if (!aligned(q, 16)) return false;
  return true;
}
// The reversible block's attention: bf16, head size 64, the same B, H, L.
static lsh_status check_rev(const lsh_problem* p, const lsh_ff_problem* f) {
  lsh_status st = check_problem(p);
  if (st != LSH_OK) return st;
  st = check_ff(f);
  if (st != LSH_OK) return st;
  if (p->B != f->B || p->H != f->H || p->L != f->L) return LSH_ERR_INVALID_ARG;
  if (p->dtype != LSH_BF16) return LSH_ERR_UNSUPPORTED;
  return LSH_OK;
}

size_t lsh_ff_workspace_size(const lsh_ff_problem* f) {
  if (check_ff(f) != LSH_OK) return 0;
  return ff_ws_bytes(*f);
}

lsh_status lsh_ff_fwd(const lsh_ff_problem* f, const void* x, const void* W1, const float* b1,
                      const void* W2, const float* b2, const void* res, void* y, void* ws,
                      size_t ws_bytes, lsh_stream_t stream) {
  lsh_status st = check_ff(f);
  if (st != LSH_OK) return st;
  if (ff_empty(f)) return LSH_OK;
  if (!x || !W1 || !b1 || !W2 || !b2 || !y) return LSH_ERR_INVALID_ARG;
  if (!all_aligned16({x, W1, b1, W2, b2, res, y}) || x == y) return LSH_ERR_INVALID_ARG;
  if (!ws || ws_bytes < ff_ws_bytes(*f) || !aligned(ws, 256)) return LSH_ERR_WORKSPACE;
  return cuda_status(launch_ff_fwd(*f, x, W1, b1, W2, b2, res, y, ws, device_status_word(),
                                   (cudaStream_t)stream));
}

lsh_status lsh_ff_bwd(const lsh_ff_problem* f, const void* x, const void* W1, const float* b1,
                      const void* W2, const float* b2, const void* dy, const void* dres,
                      const void* y_in, void* rec, void* dx, float* dW1, float* db1, float* dW2,
                      float* db2, void* ws, size_t ws_bytes, lsh_stream_t stream) {
  lsh_status st = check_ff(f);
  if (st != LSH_OK) return st;
  if (ff_empty(f)) return LSH_OK;
  if (!x || !W1 || !b1 || !W2 || !b2 || !dy || !dx || !dW1 || !db1 || !dW2 || !db2)
    return LSH_ERR_INVALID_ARG;
  if ((y_in == nullptr) != (rec == nullptr)) return LSH_ERR_INVALID_ARG;
  if (!all_aligned16({x, W1, b1, W2, b2, dy, dres, y_in, rec, dx, dW1, db1, dW2, db2}))
    return LSH_ERR_INVALID_ARG;
  if (!ws || ws_bytes < ff_ws_bytes(*f) || !aligned(ws, 256)) return LSH_ERR_WORKSPACE;
  return cuda_status(launch_ff_bwd(*f, x, W1, b1, W2, b2, dy, dres, y_in, rec, dx, dW1, db1, dW2,
                                   db2, ws, device_status_word(), (cudaStream_t)stream));
}

size_t lsh_rev_fwd_workspace_size(const lsh_problem* p, const lsh_ff_problem* f) {
  if (check_rev(p, f) != LSH_OK) return 0;
  return rev_fwd_ws_bytes(*p, *f);
}

lsh_status lsh_rev_fwd(const lsh_problem* p, const lsh_ff_problem* f, const void* x1,
                       const void* x2, const void* R, const void* W1, const float* b1,
                       const void* W2, const float* b2, void* y1, void* y2, int32_t* perm,
                       void* ws, size_t ws_bytes, lsh_stream_t stream) {
  lsh_status st = check_rev(p, f);
  if (st != LSH_OK) return st;
  if (empty(p)) return LSH_OK;
  if (!x1 || !x2 || !R || !W1 || !b1 || !W2 || !b2 || !y1 || !y2 || !perm)
    return LSH_ERR_INVALID_ARG;
  if (!all_aligned16({x1, x2, R, W1, b1, W2, b2, y1, y2})) return LSH_ERR_INVALID_ARG;
  if (!ws || ws_bytes < rev_fwd_ws_bytes(*p, *f) || !aligned(ws, 256)) return LSH_ERR_WORKSPACE;
  return cuda_status(launch_rev_fwd(*p, *f, x1, x2, R, W1, b1, W2, b2, y1, y2, perm, ws,
                                    device_status_word(), (cudaStream_t)stream));
}

size_t lsh_rev_bwd_workspace_size(const lsh_problem* p, const lsh_ff_problem* f) {
  if (check_rev(p, f) != LSH_OK) return 0;
  return rev_bwd_ws_bytes(*p, *f);
}

lsh_status lsh_rev_bwd(const lsh_problem* p, const lsh_ff_problem* f, const void* y1,
                       const void* y2, const void* dy1, const void* dy2, const int32_t* perm,
                       const void* W1, const float* b1, const void* W2, const float* b2,
                       void* x1, void* x2, void* dx1, void* dx2, float* dW1, float* db1,
                       float* dW2, float* db2, void* ws, size_t ws_bytes, lsh_stream_t stream) {
  lsh_status st = check_rev(p, f);
  if (st != LSH_OK) return st;
  if (empty(p)) return LSH_OK;
  if (!y1 || !y2 || !dy1 || !dy2 || !perm || !W1 || !b1 || !W2 || !b2 || !x1 || !x2 || !dx1 ||
      !dx2 || !dW1 || !db1 || !dW2 || !db2)
    return LSH_ERR_INVALID_ARG;
  if (!all_aligned16({y1, y2, dy1, dy2, W1, b1, W2, b2, x1, x2, dx1, dx2, dW1, db1, dW2, db2}))
    return LSH_ERR_INVALID_ARG;
  if (!ws || ws_bytes < rev_bwd_ws_bytes(*p, *f) || !aligned(ws, 256)) return LSH_ERR_WORKSPACE;
  return cuda_status(launch_rev_bwd(*p, *f, y1, y2, dy1, dy2, perm, W1, b1, W2, b2, x1, x2, dx1,
                                    dx2, dW1, db1, dW2, db2, ws, device_status_word(),
                                    (cudaStream_t)stream));
}

lsh_status lsh_device_status(lsh_stream_t stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return LSH_ERR_CUDA;
  int* w = device_status_word();
  if (!w) return LSH_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return LSH_ERR_CUDA;
  if (v != 0) {
    int z = 0;
    if (cudaMemcpy(w, &z, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return LSH_ERR_CUDA;
  }
  return (lsh_status)v;
}

lsh_status lsh_check_wait_timeout(uint64_t limit_ns, lsh_stream_t stream) {
  if (limit_ns == 0 || limit_ns > 1000000000ull) return LSH_ERR_INVALID_ARG;
  int* status = device_status_word();
  if (!status) return LSH_ERR_CUDA;
  wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(limit_ns, status);
  note_launch();
  return cuda_status(cudaGetLastError());
}

const char* lsh_status_string(lsh_status s) {
  switch (s) {
    case LSH_OK: return "ok";
    case LSH_ERR_INVALID_ARG: return "invalid argument";
    case LSH_ERR_UNSUPPORTED: return "unsupported problem (d must be 64, chunk a multiple of 64)";
    case LSH_ERR_WORKSPACE: return "workspace missing, too small or not 256-byte aligned";
    case LSH_ERR_CUDA: return "CUDA runtime error";
    case LSH_ERR_TIMEOUT: return "a kernel timed out waiting on a barrier";
    case LSH_ERR_DEVICE_CHECK: return "a kernel found an out-of-range index";
    case LSH_ERR_RANGE: return "a tensor-core-path result is not finite (a value left the fp16 range)";
  }
  return "unknown status";
}

uint64_t lsh_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
