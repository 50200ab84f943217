// LSH bucket assignment on CUDA cores (float32 fused multiply-add).
//
// "Reformer: The Efficient Transformer" (research.elamur.ai summary page),
// Key points, "LSH attention": h(x) = argmax([xR; -xR]) with a random R.
// For one rotation column k, [xR; -xR] holds s_k at index k and -s_k at index
// n_b/2 + k, so the larger of the two is |s_k| at index (s_k >= 0 ? k : n_b/2+k);
// the argmax is the largest |s_k|, lowest index on exact ties.
//
// This kernel serves float32 inputs (whose products are not exact in any
// tensor-core format) and any shape the tensor-core kernel does not cover.
#include "common.cuh"
#include "internal.h"

namespace lsh {
namespace {

constexpr int kRows = 64;  // tokens per block
constexpr int kCols = 64;  // rotation columns per tile

// Keeps (value, index) with the larger value, the smaller index on ties.
__device__ __forceinline__ void arg_better(float v, int i, float& bv, int& bi) {
  if (v > bv || (v == bv && i < bi)) { bv = v; bi = i; }
}

template <typename T>
__global__ void __launch_bounds__(256)
hash_simt_kernel(const T* __restrict__ qk, const T* __restrict__ R, int32_t* __restrict__ bucket,
                 int64_t rows, int L, int nh, int n_rounds) {
  __shared__ float xs[kRows][kD + 1];
  __shared__ float rs[kD][kCols + 1];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int r = blockIdx.y;
  const int64_t row0 = (int64_t)blockIdx.x * kRows;

  for (int e = tid; e < kRows * (kD / 4); e += 256) {
    int rr = e >> 4, c4 = (e & 15) * 4;
    float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row0 + rr < rows) f = load4(qk + (row0 + rr) * kD + c4);
    xs[rr][c4] = f.x; xs[rr][c4 + 1] = f.y; xs[rr][c4 + 2] = f.z; xs[rr][c4 + 3] = f.w;
  }
  const T* Rr = R + (int64_t)r * kD * nh;
  float best[4];
  int bidx[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) { best[i] = -1.f; bidx[i] = 0x7fffffff; }

  for (int c0 = 0; c0 < nh; c0 += kCols) {
    __syncthreads();
    for (int e = tid; e < kD * kCols; e += 256) {
      int k = e / kCols, cc = e % kCols;
      rs[k][cc] = (c0 + cc < nh) ? load1(Rr + (int64_t)k * nh + c0 + cc) : 0.f;
    }
    __syncthreads();
    float s[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) s[i][j] = 0.f;
#pragma unroll 8
    for (int k = 0; k < kD; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[ty * 4 + i][k];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = rs[k][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) s[i][j] = fmaf(a[i], b[j], s[i][j]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int col = c0 + tx + 16 * j;
      if (col < nh) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          arg_better(fabsf(s[i][j]), s[i][j] >= 0.f ? col : nh + col, best[i], bidx[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) {
      float ov = __shfl_xor_sync(0xffffffffu, best[i], o);
      int oi = __shfl_xor_sync(0xffffffffu, bidx[i], o);
      arg_better(ov, oi, best[i], bidx[i]);
    }
  }
  if (tx == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int64_t row = row0 + ty * 4 + i;
      if (row < rows) {
        int64_t bh = row / L, pos = row % L;
        bucket[(bh * n_rounds + r) * L + pos] = bidx[i];
      }
    }
  }
}

}  // namespace

cudaError_t launch_hash_simt(const lsh_problem& p, const void* qk, const void* R,
                             int32_t* bucket, cudaStream_t s) {
  const int64_t rows = (int64_t)p.B * p.H * p.L;
  dim3 grid((unsigned)((rows + kRows - 1) / kRows), (unsigned)p.n_rounds);
  const int nh = p.n_buckets / 2;
  if (p.dtype == LSH_BF16)
    hash_simt_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        (const __nv_bfloat16*)qk, (const __nv_bfloat16*)R, bucket, rows, p.L, nh, p.n_rounds);
  else
    hash_simt_kernel<float><<<grid, 256, 0, s>>>((const float*)qk, (const float*)R, bucket, rows,
                                                 p.L, nh, p.n_rounds);
  note_launch();
  return cudaGetLastError();
}

}  // namespace lsh
