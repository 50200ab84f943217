// Host-side interface between the C ABI (lsh_api.cu) and the kernel files.
#pragma once

#include <cuda_bf16.h>
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
bool launch_attn_fwd_tc_ok(const lsh_problem& p);
cudaError_t launch_attn_fwd_tc(const lsh_problem& p, const void* qk, const void* v16,
                               const int32_t* perm, void* opart_f16, float* lsepart, int* status,
                               cudaStream_t s);

// tcgen05 backward (bf16, chunk 64): forms D = dout . (out + out_lo) into D
// and fp16 copies of qk, v, dout, then writes dqk and dv (every element, the
// self-attending rows' dout included); `ws` holds bwd_tc_ws_bytes(p) bytes
// (fp16 copies, per-round fp16 partials in token order, edge map).
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

// ---- dense products of the feed-forward layer (tcgen05) -------------------
// An operand of C = A B: mn_major = stored [K][rows] (else [rows][K]); heads =
// the attention's [B, H, L, 64] layout read as token rows b L + l with 64 H
// columns (else a plain row-major matrix of rows x cols); row0 = first row
// (tokens for the head layout, K rows when mn_major) of this product.
struct GemmOpDev {
  int mn_major, heads, L;
  int64_t row0;
};
struct GemmOpHost {
  const void* base;
  int mn_major, heads;
  int64_t rows, cols;   // plain matrix extent
  int L, H, B;          // head layout extent
  int64_t row0;
};
// Epilogue, per element (row, column c) of the M x N result:
//   v = acc + bias[c]; v = max(v, 0) if relu; v = 0 unless mask[row][c] > 0;
//   v = res + res_sign * v where res is given (same layout as the output);
//   out (bf16, or fp32 with optional accumulate) at row0 + row.
struct GemmEpi {
  const float* bias;
  int relu;
  const __nv_bfloat16* mask;
  int64_t ldm;
  const __nv_bfloat16* res;
  float res_sign;
  void* out;
  int out_f32, accumulate, out_heads;
  int64_t ldo, row0;
  int L, H;
  int M;
  // optional scratch of kGemmMaxSplits * M * N floats: a plain float32
  // product with few tiles is then split along K (the splits' sums are added
  // in a fixed order, so the result stays deterministic)
  float* split_part;
};
constexpr int kGemmMaxSplits = 4;
// K a multiple of 64, N a multiple of 64; rows past M are neither read into
// the output nor written.
cudaError_t launch_gemm_tc(const GemmOpHost& a, const GemmOpHost& b, int M, int N, int K,
                           const GemmEpi& e, int* status, cudaStream_t s);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---- chunked feed-forward and the reversible block (rev_block.cu) ----------
size_t ff_ws_bytes(const lsh_ff_problem& f);
cudaError_t launch_ff_fwd(const lsh_ff_problem& f, const void* x, const void* W1, const float* b1,
                          const void* W2, const float* b2, const void* res, void* y, void* ws,
                          int* status, cudaStream_t s);
cudaError_t launch_ff_bwd(const lsh_ff_problem& f, const void* x, const void* W1, const float* b1,
                          const void* W2, const float* b2, const void* dy, const void* dres,
                          const void* y_in, void* rec, void* dx, float* dW1, float* db1,
                          float* dW2, float* db2, void* ws, int* status, cudaStream_t s);
size_t rev_fwd_ws_bytes(const lsh_problem& p, const lsh_ff_problem& f);
size_t rev_bwd_ws_bytes(const lsh_problem& p, const lsh_ff_problem& f);
cudaError_t launch_rev_fwd(const lsh_problem& p, const lsh_ff_problem& f, const void* x1,
                           const void* x2, const void* R, const void* W1, const float* b1,
                           const void* W2, const float* b2, void* y1, void* y2, int32_t* perm,
                           void* ws, int* status, cudaStream_t s);
cudaError_t launch_rev_bwd(const lsh_problem& p, const lsh_ff_problem& f, const void* y1,
                           const void* y2, const void* dy1, const void* dy2, const int32_t* perm,
                           const void* W1, const float* b1, const void* W2, const float* b2,
                           void* x1, void* x2, void* dx1, void* dx2, float* dW1, float* db1,
                           float* dW2, float* db2, void* ws, int* status, cudaStream_t s);

}  // namespace lsh
