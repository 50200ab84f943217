// The layer around the attention: a position-wise feed-forward run chunk by
// chunk, and the reversible residual block that joins it to LSH attention
// ("Reformer: The Efficient Transformer", research.elamur.ai summary page,
// Key points, "Reversible layers": reversible residual layers after Gomez et
// al. 2017 recompute a layer's inputs from its outputs in the backward pass;
// the feed-forward runs in chunks, which leaves its results unchanged).
//
//   G(x) = max(0, x W1 + b1) W2 + b2           (per position)
//   y1 = x1 + F(x2),  y2 = x2 + G(y1)           F = LSH attention, qk = v = x2
//   x2 = y2 - G(y1),  x1 = y1 - F(x2)           (backward, from the outputs)
//
// Activations are the attention's [B, H, L, 64] bf16 arrays; token (b, l)
// has d_model = 64 H features, its H head rows side by side. The
// feed-forward's products run on the tensor cores (gemm_tc.cu), ff_chunk
// positions at a time, so only a [ff_chunk, d_ff] hidden block exists at
// once; the bias sums are formed in a fixed order, so every result is
// deterministic.
#include <cuda_bf16.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace lsh {
namespace {

__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// y = a + sign * (o + o_lo) elementwise (o_lo may be null), 8 values a thread.
__global__ void __launch_bounds__(256)
add_out_kernel(const __nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ o,
               const __nv_bfloat16* __restrict__ o_lo, float sign, __nv_bfloat16* __restrict__ y,
               int64_t n8) {
  const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= n8) return;
  const uint4 ua = __ldg(reinterpret_cast<const uint4*>(a) + k);
  const uint4 uo = __ldg(reinterpret_cast<const uint4*>(o) + k);
  const uint4 ul = o_lo ? __ldg(reinterpret_cast<const uint4*>(o_lo) + k) : make_uint4(0u, 0u, 0u, 0u);
  const uint32_t A[4] = {ua.x, ua.y, ua.z, ua.w}, O[4] = {uo.x, uo.y, uo.z, uo.w};
  const uint32_t Lo[4] = {ul.x, ul.y, ul.z, ul.w};
  uint32_t r[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    r[i] = pack_bf2(fmaf(sign, bf_lo(O[i]) + bf_lo(Lo[i]), bf_lo(A[i])),
                    fmaf(sign, bf_hi(O[i]) + bf_hi(Lo[i]), bf_hi(A[i])));
  reinterpret_cast<uint4*>(y)[k] = make_uint4(r[0], r[1], r[2], r[3]);
}

// out = a + g1 + g2 (a bf16, g1 and g2 fp32), 8 values a thread.
__global__ void __launch_bounds__(256)
sum3_kernel(const __nv_bfloat16* __restrict__ a, const float* __restrict__ g1,
            const float* __restrict__ g2, __nv_bfloat16* __restrict__ out, int64_t n8) {
  const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= n8) return;
  const uint4 ua = __ldg(reinterpret_cast<const uint4*>(a) + k);
  const uint32_t A[4] = {ua.x, ua.y, ua.z, ua.w};
  const float4* p1 = reinterpret_cast<const float4*>(g1) + 2 * k;
  const float4* p2 = reinterpret_cast<const float4*>(g2) + 2 * k;
  const float4 a1 = __ldg(p1), b1 = __ldg(p1 + 1), a2 = __ldg(p2), b2 = __ldg(p2 + 1);
  const float s[8] = {a1.x + a2.x, a1.y + a2.y, a1.z + a2.z, a1.w + a2.w,
                      b1.x + b2.x, b1.y + b2.y, b1.z + b2.z, b1.w + b2.w};
  uint32_t r[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) r[i] = pack_bf2(bf_lo(A[i]) + s[2 * i], bf_hi(A[i]) + s[2 * i + 1]);
  reinterpret_cast<uint4*>(out)[k] = make_uint4(r[0], r[1], r[2], r[3]);
}

// Column sums of a bf16 block, in two deterministic passes.
// src(row, c) is a plain [*, ld] matrix or the head layout (token rows, 64 H
// columns, row g = b L + l). Pass 1: block (x, y) takes 256 columns and the
// kSumRows rows starting at y kSumRows; warp w of it adds rows w, w + 8, ...
// (16-byte loads, 8 columns a thread), then the 8 warps' sums are added in
// warp order into part[y][c]. Pass 2: db[c] (+)= the parts in y order.
constexpr int kSumRows = 256, kSumU = 8;

__global__ void __launch_bounds__(256)
colsum_part_kernel(const __nv_bfloat16* __restrict__ src, int heads, int64_t r0, int rows, int N,
                   int64_t ld, int L, int H, float* __restrict__ part) {
  __shared__ float red[8][256];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int c = blockIdx.x * 256 + lane * 8;
  const int lo = blockIdx.y * kSumRows, hi = min(rows, lo + kSumRows);
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  if (c < N) {
    // kSumU rows' loads in flight per thread before any of them is added;
    // the adds still run in row order
    for (int r = lo + w; r < hi; r += 8 * kSumU) {
      uint4 u[kSumU];
#pragma unroll
      for (int j = 0; j < kSumU; ++j) {
        const int rr = r + 8 * j;
        if (rr < hi) {
          const int64_t g = r0 + rr;
          int64_t off;
          if (heads) {
            const int64_t b = g / L, l = g - b * L;
            off = ((b * H + c / 64) * L + l) * 64 + (c & 63);
          } else {
            off = g * ld + c;
          }
          u[j] = __ldg(reinterpret_cast<const uint4*>(src + off));
        }
      }
#pragma unroll
      for (int j = 0; j < kSumU; ++j) {
        if (r + 8 * j < hi) {
          const uint32_t v[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc[2 * i] += bf_lo(v[i]);
            acc[2 * i + 1] += bf_hi(v[i]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) red[w][lane * 8 + i] = acc[i];
  __syncthreads();
  const int cc = blockIdx.x * 256 + threadIdx.x;
  if (cc < N) {
    float t = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) t += red[k][threadIdx.x];
    part[(int64_t)blockIdx.y * N + cc] = t;
  }
}

__global__ void __launch_bounds__(256)
colsum_final_kernel(const float* __restrict__ part, int S, int N, float* __restrict__ db,
                    int accumulate) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= N) return;
  float t = 0.f;
  for (int k = 0; k < S; ++k) t += part[(int64_t)k * N + c];
  db[c] = accumulate ? db[c] + t : t;
}

cudaError_t colsum(const __nv_bfloat16* src, int heads, int64_t r0, int rows, int N, int64_t ld,
                   int L, int H, float* part, float* db, bool accumulate, cudaStream_t s) {
  const int S = (rows + kSumRows - 1) / kSumRows;
  colsum_part_kernel<<<dim3((unsigned)((N + 255) / 256), (unsigned)S), 256, 0, s>>>(
      src, heads, r0, rows, N, ld, L, H, part);
  colsum_final_kernel<<<(unsigned)((N + 255) / 256), 256, 0, s>>>(part, S, N, db,
                                                                  accumulate ? 1 : 0);
  note_launch(2);
  return cudaGetLastError();
}

GemmOpHost heads_op(const void* base, const lsh_ff_problem& f, int mn_major, int64_t row0) {
  GemmOpHost o{};
  o.base = base;
  o.mn_major = mn_major;
  o.heads = 1;
  o.L = f.L;
  o.H = f.H;
  o.B = f.B;
  o.row0 = row0;
  return o;
}
GemmOpHost plain_op(const void* base, int64_t rows, int64_t cols, int mn_major) {
  GemmOpHost o{};
  o.base = base;
  o.mn_major = mn_major;
  o.heads = 0;
  o.rows = rows;
  o.cols = cols;
  return o;
}
GemmEpi epi() {
  GemmEpi e{};
  e.res_sign = 1.f;
  return e;
}

struct FfWs {
  __nv_bfloat16* h;    // [ff_chunk, d_ff] hidden block
  __nv_bfloat16* dh;   // [ff_chunk, d_ff] its gradient
  float* part;         // partial column sums of the bias gradients
  float* split;        // K-split partial sums of the weight gradients
};
size_t ff_part_bytes(const lsh_ff_problem& f) {
  const size_t S = ((size_t)f.ff_chunk + kSumRows - 1) / kSumRows;
  return align_up(S * (size_t)std::max(f.d_ff, 64 * f.H) * 4, 256);
}
size_t ff_split_bytes(const lsh_ff_problem& f) {
  return align_up((size_t)kGemmMaxSplits * 64 * f.H * f.d_ff * 4, 256);
}
FfWs ff_carve(const lsh_ff_problem& f, void* ws) {
  FfWs w;
  const size_t hb = align_up((size_t)f.ff_chunk * f.d_ff * 2, 256);
  w.h = (__nv_bfloat16*)ws;
  w.dh = (__nv_bfloat16*)((char*)ws + hb);
  w.part = (float*)((char*)ws + 2 * hb);
  w.split = (float*)((char*)ws + 2 * hb + ff_part_bytes(f));
  return w;
}

// h = max(0, x[r0 .. r0+Mc) W1 + b1)
cudaError_t ff_hidden(const lsh_ff_problem& f, const void* x, const void* W1, const float* b1,
                      __nv_bfloat16* h, int64_t r0, int Mc, int* status, cudaStream_t s) {
  const int D = 64 * f.H;
  GemmEpi e = epi();
  e.bias = b1;
  e.relu = 1;
  e.out = h;
  e.ldo = f.d_ff;
  e.M = Mc;
  return launch_gemm_tc(heads_op(x, f, 0, r0), plain_op(W1, D, f.d_ff, 1), Mc, f.d_ff, D, e,
                        status, s);
}

// out[r0 ..] = res + sign * (h W2 + b2)   (res may be null)
cudaError_t ff_out(const lsh_ff_problem& f, const __nv_bfloat16* h, const void* W2, const float* b2,
                   const void* res, float sign, void* out, int64_t r0, int Mc, int* status,
                   cudaStream_t s) {
  const int D = 64 * f.H;
  GemmEpi e = epi();
  e.bias = b2;
  e.res = (const __nv_bfloat16*)res;
  e.res_sign = sign;
  e.out = out;
  e.out_heads = 1;
  e.row0 = r0;
  e.L = f.L;
  e.H = f.H;
  e.M = Mc;
  return launch_gemm_tc(plain_op(h, Mc, f.d_ff, 0), plain_op(W2, f.d_ff, D, 1), Mc, D, f.d_ff, e,
                        status, s);
}

}  // namespace

size_t ff_ws_bytes(const lsh_ff_problem& f) {
  return 2 * align_up((size_t)f.ff_chunk * f.d_ff * 2, 256) + ff_part_bytes(f) + ff_split_bytes(f);
}

cudaError_t launch_ff_fwd(const lsh_ff_problem& f, const void* x, const void* W1, const float* b1,
                          const void* W2, const float* b2, const void* res, void* y, void* ws,
                          int* status, cudaStream_t s) {
  const FfWs w = ff_carve(f, ws);
  const int64_t T = (int64_t)f.B * f.L;
  for (int64_t r0 = 0; r0 < T; r0 += f.ff_chunk) {
    const int Mc = (int)std::min<int64_t>(f.ff_chunk, T - r0);
    cudaError_t e = ff_hidden(f, x, W1, b1, w.h, r0, Mc, status, s);
    if (e != cudaSuccess) return e;
    e = ff_out(f, w.h, W2, b2, res, 1.f, y, r0, Mc, status, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_ff_bwd(const lsh_ff_problem& f, const void* x, const void* W1, const float* b1,
                          const void* W2, const float* b2, const void* dy, const void* dres,
                          const void* y_in, void* rec, void* dx, float* dW1, float* db1,
                          float* dW2, float* db2, void* ws, int* status, cudaStream_t s) {
  const FfWs w = ff_carve(f, ws);
  const int64_t T = (int64_t)f.B * f.L;
  const int D = 64 * f.H;
  for (int64_t r0 = 0; r0 < T; r0 += f.ff_chunk) {
    const int Mc = (int)std::min<int64_t>(f.ff_chunk, T - r0);
    const bool acc = r0 > 0;
    cudaError_t e = ff_hidden(f, x, W1, b1, w.h, r0, Mc, status, s);
    if (e != cudaSuccess) return e;
    if (rec) {
      // the reversible block's reconstruction y_in - G(x)
      e = ff_out(f, w.h, W2, b2, y_in, -1.f, rec, r0, Mc, status, s);
      if (e != cudaSuccess) return e;
    }
    {
      // dh = (dy W2^T) * [h > 0]
      GemmEpi ep = epi();
      ep.mask = w.h;
      ep.ldm = f.d_ff;
      ep.out = w.dh;
      ep.ldo = f.d_ff;
      ep.M = Mc;
      e = launch_gemm_tc(heads_op(dy, f, 0, r0), plain_op(W2, f.d_ff, D, 0), Mc, f.d_ff, D, ep,
                         status, s);
      if (e != cudaSuccess) return e;
    }
    {
      // dW2 (+)= h^T dy
      GemmEpi ep = epi();
      ep.out = dW2;
      ep.out_f32 = 1;
      ep.accumulate = acc;
      ep.ldo = D;
      ep.M = f.d_ff;
      ep.split_part = w.split;
      e = launch_gemm_tc(plain_op(w.h, Mc, f.d_ff, 1), heads_op(dy, f, 1, r0), f.d_ff, D, Mc, ep,
                         status, s);
      if (e != cudaSuccess) return e;
    }
    {
      // dW1 (+)= x^T dh
      GemmEpi ep = epi();
      ep.out = dW1;
      ep.out_f32 = 1;
      ep.accumulate = acc;
      ep.ldo = f.d_ff;
      ep.M = D;
      ep.split_part = w.split;
      e = launch_gemm_tc(heads_op(x, f, 1, r0), plain_op(w.dh, Mc, f.d_ff, 1), D, f.d_ff, Mc, ep,
                         status, s);
      if (e != cudaSuccess) return e;
    }
    {
      // dx = dres + dh W1^T
      GemmEpi ep = epi();
      ep.res = (const __nv_bfloat16*)dres;
      ep.out = dx;
      ep.out_heads = 1;
      ep.row0 = r0;
      ep.L = f.L;
      ep.H = f.H;
      ep.M = Mc;
      e = launch_gemm_tc(plain_op(w.dh, Mc, f.d_ff, 0), plain_op(W1, D, f.d_ff, 0), Mc, D, f.d_ff,
                         ep, status, s);
      if (e != cudaSuccess) return e;
    }
    e = colsum(w.dh, 0, 0, Mc, f.d_ff, f.d_ff, f.L, f.H, w.part, db1, acc, s);
    if (e != cudaSuccess) return e;
    e = colsum((const __nv_bfloat16*)dy, 1, r0, Mc, D, 0, f.L, f.H, w.part, db2, acc, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// ---------------------------------------------------------------- block
namespace {
struct RevFwdWs {
  int32_t* bucket;
  SortWs sort;
  __nv_bfloat16 *out, *out_lo;
  float* lse;
  void* fwd;
  void* ff;
  size_t bytes;
};
RevFwdWs rev_fwd_carve(const lsh_problem& p, const lsh_ff_problem& f, void* base) {
  const size_t N = (size_t)p.B * p.H * p.L;
  char* c = (char*)base;
  size_t off = 0;
  RevFwdWs w{};
  w.bucket = (int32_t*)(c + off);
  off += align_up(N * p.n_rounds * 4, 256);
  void* sort_base = c + off;
  off += align_up(sort_ws_bytes(p), 256);
  w.out = (__nv_bfloat16*)(c + off);
  off += align_up(N * 64 * 2, 256);
  w.out_lo = (__nv_bfloat16*)(c + off);
  off += align_up(N * 64 * 2, 256);
  w.lse = (float*)(c + off);
  off += align_up(N * 4, 256);
  w.fwd = c + off;
  off += align_up(fwd_ws_bytes(p), 256);
  w.ff = c + off;
  off += align_up(ff_ws_bytes(f), 256);
  w.bytes = off;
  if (base) w.sort = sort_ws_carve(p, sort_base);
  return w;
}
struct RevBwdWs {
  __nv_bfloat16 *out, *out_lo;
  float* lse;
  void* fwd;
  void* bwd;
  float *dqk, *dv;
  void* ff;
  size_t bytes;
};
RevBwdWs rev_bwd_carve(const lsh_problem& p, const lsh_ff_problem& f, void* base) {
  const size_t N = (size_t)p.B * p.H * p.L;
  char* c = (char*)base;
  size_t off = 0;
  RevBwdWs w{};
  w.out = (__nv_bfloat16*)(c + off);
  off += align_up(N * 64 * 2, 256);
  w.out_lo = (__nv_bfloat16*)(c + off);
  off += align_up(N * 64 * 2, 256);
  w.lse = (float*)(c + off);
  off += align_up(N * 4, 256);
  w.fwd = c + off;
  off += align_up(fwd_ws_bytes(p), 256);
  w.bwd = c + off;
  off += align_up(bwd_ws_bytes(p), 256);
  w.dqk = (float*)(c + off);
  off += align_up(N * 64 * 4, 256);
  w.dv = (float*)(c + off);
  off += align_up(N * 64 * 4, 256);
  w.ff = c + off;
  off += align_up(ff_ws_bytes(f), 256);
  w.bytes = off;
  return w;
}

cudaError_t add_out(const void* a, const void* o, const void* o_lo, float sign, void* y, int64_t N,
                    cudaStream_t s) {
  const int64_t n8 = N * 8;
  add_out_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, s>>>(
      (const __nv_bfloat16*)a, (const __nv_bfloat16*)o, (const __nv_bfloat16*)o_lo, sign,
      (__nv_bfloat16*)y, n8);
  note_launch();
  return cudaGetLastError();
}
}  // namespace

size_t rev_fwd_ws_bytes(const lsh_problem& p, const lsh_ff_problem& f) {
  return rev_fwd_carve(p, f, nullptr).bytes;
}
size_t rev_bwd_ws_bytes(const lsh_problem& p, const lsh_ff_problem& f) {
  return rev_bwd_carve(p, f, nullptr).bytes;
}

cudaError_t launch_rev_fwd(const lsh_problem& p, const lsh_ff_problem& f, const void* x1,
                           const void* x2, const void* R, const void* W1, const float* b1,
                           const void* W2, const float* b2, void* y1, void* y2, int32_t* perm,
                           void* ws, int* status, cudaStream_t s) {
  const RevFwdWs w = rev_fwd_carve(p, f, ws);
  const int64_t N = (int64_t)p.B * p.H * p.L;
  cudaError_t e = launch_hash_tc(p, x2, R, w.bucket, status, s);
  if (e == cudaErrorNotSupported) e = launch_hash_simt(p, x2, R, w.bucket, s);
  if (e != cudaSuccess) return e;
  e = launch_sort(p, w.bucket, perm, w.sort, status, s);
  if (e != cudaSuccess) return e;
  e = launch_attn_fwd(p, x2, x2, perm, w.out, w.out_lo, w.lse, fwd_ws_carve(p, w.fwd), status, s);
  if (e != cudaSuccess) return e;
  e = add_out(x1, w.out, w.out_lo, 1.f, y1, N, s);
  if (e != cudaSuccess) return e;
  return launch_ff_fwd(f, y1, W1, b1, W2, b2, x2, y2, w.ff, status, s);
}

cudaError_t launch_rev_bwd(const lsh_problem& p, const lsh_ff_problem& f, const void* y1,
                           const void* y2, const void* dy1, const void* dy2, const int32_t* perm,
                           const void* W1, const float* b1, const void* W2, const float* b2,
                           void* x1, void* x2, void* dx1, void* dx2, float* dW1, float* db1,
                           float* dW2, float* db2, void* ws, int* status, cudaStream_t s) {
  const RevBwdWs w = rev_bwd_carve(p, f, ws);
  const int64_t N = (int64_t)p.B * p.H * p.L;
  // G half: x2 = y2 - G(y1), dx1 = dz1 = dy1 + (dG/dy1)^T dy2, G's weight gradients
  cudaError_t e = launch_ff_bwd(f, y1, W1, b1, W2, b2, dy2, dy1, y2, x2, dx1, dW1, db1, dW2, db2,
                                w.ff, status, s);
  if (e != cudaSuccess) return e;
  // F half: x1 = y1 - F(x2), dx2 = dy2 + (dF/dx2)^T dz1 (x2 is both qk and v)
  e = launch_attn_fwd(p, x2, x2, perm, w.out, w.out_lo, w.lse, fwd_ws_carve(p, w.fwd), status, s);
  if (e != cudaSuccess) return e;
  e = add_out(y1, w.out, w.out_lo, -1.f, x1, N, s);
  if (e != cudaSuccess) return e;
  e = launch_attn_bwd(p, x2, x2, perm, w.out, w.out_lo, w.lse, dx1, w.dqk, w.dv, w.bwd, status, s);
  if (e != cudaSuccess) return e;
  const int64_t n8 = N * 8;
  sum3_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, s>>>(
      (const __nv_bfloat16*)dy2, w.dqk, w.dv, (__nv_bfloat16*)dx2, n8);
  note_launch();
  return cudaGetLastError();
}

}  // namespace lsh
