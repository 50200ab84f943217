// Host-side interface between the C ABI (lsh_api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "lsh.h"

namespace lsh {

constexpr int kDHead = 64;  // the only head size the kernels support

// Counts one kernel launch (for lsh_launch_count()).
void note_launch(int n = 1);

// Device status word of the current device (LSH_OK until a kernel records a
// timeout or an index check); nullptr if it cannot be resolved.
int* device_status_word();

// ---- hashing ----
cudaError_t launch_hash_simt(const lsh_problem& p, const void* qk, const void* R,
                             int32_t* bucket, cudaStream_t s);
// tcgen05 path (bf16 inputs); returns cudaErrorNotSupported when the shape
// does not suit it, so the caller can choose the SIMT kernel instead.
cudaError_t launch_hash_tc(const lsh_problem& p, const void* qk, const void* R,
                           int32_t* bucket, int* status, cudaStream_t s);

// ---- sorting ----
struct SortWs {
  uint32_t* sorted;   // [S * L] tile-sorted packed keys
  int32_t* counts;    // [S * n_buckets * tiles]
  int32_t* base;      // [S * n_buckets]
};
size_t sort_ws_bytes(const lsh_problem& p);
SortWs sort_ws_carve(const lsh_problem& p, void* ws);
cudaError_t launch_sort(const lsh_problem& p, const int32_t* bucket, int32_t* perm,
                        const SortWs& ws, int* status, cudaStream_t s);

// ---- attention ----
struct FwdWs {
  float* opart;    // [n_rounds, B*H*L, d] per-round outputs, original order
  float* lsepart;  // [n_rounds, B*H*L] per-round log-sum-exps
};
size_t fwd_ws_bytes(const lsh_problem& p);
FwdWs fwd_ws_carve(const lsh_problem& p, void* ws);
cudaError_t launch_attn_fwd(const lsh_problem& p, const void* qk, const void* v,
                            const int32_t* perm, void* out, void* out_lo, float* lse, const FwdWs& ws,
                            int* status, cudaStream_t s);

// tcgen05 per-round forward (bf16, chunk 64): writes fp16 per-round outputs
// [n_rounds][B*H*L][64] and lse_r; cudaErrorNotSupported for other shapes.
cudaError_t launch_attn_fwd_tc(const lsh_problem& p, const void* qk, const void* v,
                               const int32_t* perm, void* opart_f16, float* lsepart, int* status,
                               cudaStream_t s);

// tcgen05 backward (bf16, chunk 64): forms D = dout . (out + out_lo) into D
// and fp16 copies of qk, v, dout, then writes dqk and dv (every element, the
// self-attending rows' dout included); `ws` holds bwd_tc_ws_bytes(p) bytes
// (fp16 copies, inverse permutation, per-round fp16 partials).
// bwd_tc_ws_bytes is 0 and the launcher returns cudaErrorNotSupported for
// other problems.
size_t bwd_tc_ws_bytes(const lsh_problem& p);
cudaError_t launch_attn_bwd_tc(const lsh_problem& p, const void* qk, const void* v,
                               const void* dout, const void* out, const void* out_lo,
                               const int32_t* perm, const float* lse, float* D, float* dqk,
                               float* dv, void* ws, int* status, cudaStream_t s);

size_t bwd_ws_bytes(const lsh_problem& p);
cudaError_t launch_attn_bwd(const lsh_problem& p, const void* qk, const void* v,
                            const int32_t* perm, const void* out, const void* out_lo,
                            const float* lse, const void* dout, float* dqk, float* dv, void* ws,
                            int* status, cudaStream_t s);

// ---- local attention (identity order, n_back / n_fwd chunks of overlap) ----
size_t local_fwd_ws_bytes(const lsh_problem& p, int n_back, int n_fwd);
cudaError_t launch_local_fwd(const lsh_problem& p, int n_back, int n_fwd, const void* qk,
                             const void* v, void* out, void* out_lo, float* lse, void* ws,
                             int* status, cudaStream_t s);
size_t local_bwd_ws_bytes(const lsh_problem& p, int n_back, int n_fwd);
cudaError_t launch_local_bwd(const lsh_problem& p, int n_back, int n_fwd, const void* qk,
                             const void* v, const void* out, const void* out_lo, const float* lse,
                             const void* dout, float* dqk, float* dv, void* ws, int* status,
                             cudaStream_t s);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace lsh
