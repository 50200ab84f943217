// Chunked LSH attention on CUDA cores: per-round forward, round combine,
// and the recomputing backward pass. Serves float32 inputs and every shape.
//
// "Reformer: The Efficient Transformer" (research.elamur.ai summary page):
//  - Key points, "LSH attention": after sorting, each chunk of m positions
//    attends to itself and the chunk before it;
//  - Key points, "Shared-QK Transformer": keys are the queries; a token does
//    not attend to itself unless it has no other valid target;
//  - Key points, "Number of hash rounds": several rounds; here they are
//    combined by a softmax over their per-round log-sum-exps;
//  - Summary: activations are recomputed instead of stored, which is what the
//    backward does with the attention weights.
//
// Block = 64 sorted query slots of one (batch, head, round) segment; the
// key window [max(0,(c-1)m), (c+1)m) is walked in tiles of 64 keys.
// Thread (ty, tx) of a 16x16 grid owns rows ty*4+i and columns tx+16j.
#include "common.cuh"
#include "internal.h"

namespace lsh {
// bf16 pair -> fp16 pair (exact inside the fp16 range)
__device__ __forceinline__ uint32_t tc_bf16x2_to_f16x2(uint32_t u) {
  const float lo = __uint_as_float(u << 16), hi = __uint_as_float(u & 0xffff0000u);
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
}  // namespace lsh

namespace lsh {
namespace {

constexpr int kQ = 64;    // query rows per block
constexpr int kK = 64;    // keys per tile
constexpr int kP = kD + 1;  // padded shared-memory row (floats)

// Reads perm[i] (the identity order when pr is null); an id outside [0, L) is
// recorded in the status word and replaced by 0 so that no gather leaves the
// tensor.
__device__ __forceinline__ int checked_pos(const int32_t* pr, int i, int L, int* status) {
  if (!pr) return i;
  int q = pr[i];
  if ((unsigned)q >= (unsigned)L) {
    record_status(status, (int)LSH_ERR_DEVICE_CHECK);
    q = 0;
  }
  return q;
}

template <typename T>
__device__ __forceinline__ void load_rows(float (*dst)[kP], const T* __restrict__ base,
                                          const int* pos, int tid) {
  for (int e = tid; e < kK * (kD / 4); e += 256) {
    int row = e >> 4, c4 = (e & 15) * 4;
    float4 f = load4(base + (int64_t)pos[row] * kD + c4);
    dst[row][c4] = f.x; dst[row][c4 + 1] = f.y; dst[row][c4 + 2] = f.z; dst[row][c4 + 3] = f.w;
  }
}

// Per-round forward. Writes o_r (normalised) and lse_r in original order.
// The queries of sorted chunk c see the key slots of chunks [c - n_back,
// c + n_fwd] (clipped to the segment): n_back = 1, n_fwd = 0 is the LSH
// window; a null perm is the identity order (local attention).
template <typename T>
__global__ void __launch_bounds__(256)
fwd_round_kernel(const T* __restrict__ qk, const T* __restrict__ v, const int32_t* __restrict__ perm,
                 float* __restrict__ opart, float* __restrict__ lsepart, int L, int m,
                 int n_rounds, int64_t N, int causal, float scale_log2, int n_back, int n_fwd,
                 int* status) {
  extern __shared__ float smem[];
  float(*Qs)[kP] = reinterpret_cast<float(*)[kP]>(smem);
  float(*Ks)[kP] = Qs + kQ;
  float(*Vs)[kP] = Ks + kK;
  float(*Ps)[kP] = Vs + kK;
  int* qpos = reinterpret_cast<int*>(Ps + kQ);
  int* kpos = qpos + kQ;

  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int qblocks = L / kQ;
  const int qb = blockIdx.x % qblocks;
  const int64_t seg = blockIdx.x / qblocks;
  const int r = (int)(seg % n_rounds);
  const int64_t bh = seg / n_rounds;
  const int32_t* pr = perm ? perm + seg * L : nullptr;
  const T* X = qk + bh * L * kD;
  const T* Vb = v + bh * L * kD;
  const int t0 = qb * kQ, c = t0 / m;
  const int k_lo = (int)max((int64_t)0, (int64_t)(c - n_back) * m);
  const int k_hi = (int)min((int64_t)L, (int64_t)(c + 1 + n_fwd) * m);

  if (tid < kQ) qpos[tid] = checked_pos(pr, t0 + tid, L, status);
  __syncthreads();
  load_rows(Qs, X, qpos, tid);
  int myq[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) myq[i] = qpos[ty * 4 + i];

  float mrow[4], lrow[4], acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    mrow[i] = -INFINITY; lrow[i] = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  }

  for (int kt = k_lo; kt < k_hi; kt += kK) {
    __syncthreads();
    if (tid < kK) kpos[tid] = checked_pos(pr, kt + tid, L, status);
    __syncthreads();
    load_rows(Ks, X, kpos, tid);
    load_rows(Vs, Vb, kpos, tid);
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
      for (int i = 0; i < 4; ++i) a[i] = Qs[ty * 4 + i][k];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Ks[tx + 16 * j][k];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) s[i][j] = fmaf(a[i], b[j], s[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float tmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        int kp = kpos[tx + 16 * j];
        bool ok = (kp != myq[i]) && (!causal || kp < myq[i]);
        s[i][j] = ok ? s[i][j] * scale_log2 : -INFINITY;
        tmax = fmaxf(tmax, s[i][j]);
      }
      tmax = warp_max16(tmax);
      float mnew = fmaxf(mrow[i], tmax);
      float msafe = (mnew == -INFINITY) ? 0.f : mnew;
      float alpha = exp2f(mrow[i] - msafe);
      float rs = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float pv = exp2f(s[i][j] - msafe);
        Ps[ty * 4 + i][tx + 16 * j] = pv;
        rs += pv;
      }
      rs = warp_sum16(rs);
      lrow[i] = lrow[i] * alpha + rs;
      mrow[i] = mnew;
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] *= alpha;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kK; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = Ps[ty * 4 + i][k];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Vs[k][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t row = (int64_t)r * N + bh * L + myq[i];
    const bool has = lrow[i] > 0.f;
    const float inv = has ? 1.f / lrow[i] : 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) opart[row * kD + tx + 16 * j] = acc[i][j] * inv;
    if (tx == 0) lsepart[row] = has ? (mrow[i] + log2f(lrow[i])) * kLn2 : -INFINITY;
  }
}

// Round combine in original order; 16 threads per token, 4 columns each.
// PT: type of the per-round outputs (float from the CUDA-core kernel, __half
// from the tensor-core kernel).
template <typename T, typename PT>
__global__ void __launch_bounds__(256)
combine_kernel(const PT* __restrict__ opart, const float* __restrict__ lsepart,
               const T* __restrict__ v, T* __restrict__ out, T* __restrict__ out_lo,
               float* __restrict__ lse, int64_t N, int n_rounds) {
  const int64_t tok = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 4;
  const int c4 = (threadIdx.x & 15) * 4;
  if (tok >= N) return;
  float mx = -INFINITY;
  for (int r = 0; r < n_rounds; ++r) mx = fmaxf(mx, lsepart[(int64_t)r * N + tok]);
  if (mx == -INFINITY) {
    store4(out + tok * kD + c4, load4(v + tok * kD + c4));
    if (out_lo) store4(out_lo + tok * kD + c4, make_float4(0.f, 0.f, 0.f, 0.f));
    if (c4 == 0) lse[tok] = -INFINITY;
    return;
  }
  float tot = 0.f;
  for (int r = 0; r < n_rounds; ++r) tot += expf(lsepart[(int64_t)r * N + tok] - mx);
  const float LSE = mx + logf(tot);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int r = 0; r < n_rounds; ++r) {
    float l = lsepart[(int64_t)r * N + tok];
    if (l == -INFINITY) continue;
    float w = expf(l - LSE);
    float4 o = load4(opart + ((int64_t)r * N + tok) * kD + c4);
    acc.x += w * o.x; acc.y += w * o.y; acc.z += w * o.z; acc.w += w * o.w;
  }
  store4(out + tok * kD + c4, acc);
  if (out_lo) {
    float4 hi = load4(out + tok * kD + c4);   // the rounded value just stored
    store4(out_lo + tok * kD + c4, make_float4(acc.x - hi.x, acc.y - hi.y, acc.z - hi.z,
                                               acc.w - hi.w));
  }
  if (c4 == 0) lse[tok] = LSE;
}

// Round combine for fp16 per-round outputs (tensor-core forward): 8 threads
// per token, 8 columns each (16-byte loads and stores); round loads are
// unrolled so several are in flight.
__device__ __forceinline__ void unpack8(uint4 u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ uint4 pack8_bf16(const float* f) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__global__ void __launch_bounds__(256)
combine_f16_kernel(const __half* __restrict__ opart, const float* __restrict__ lsepart,
                   const __nv_bfloat16* __restrict__ v, __nv_bfloat16* __restrict__ out,
                   __nv_bfloat16* __restrict__ out_lo, float* __restrict__ lse, int64_t N,
                   int n_rounds, int* status) {
  const int64_t tok = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 3;
  const int c8 = (threadIdx.x & 7) * 8;
  if (tok >= N) return;
  float mx = -INFINITY;
  for (int r = 0; r < n_rounds; ++r) mx = fmaxf(mx, __ldg(lsepart + (int64_t)r * N + tok));
  uint4* o16 = reinterpret_cast<uint4*>(out + tok * kD + c8);
  if (mx == -INFINITY) {
    *o16 = *reinterpret_cast<const uint4*>(v + tok * kD + c8);
    if (out_lo) *reinterpret_cast<uint4*>(out_lo + tok * kD + c8) = make_uint4(0u, 0u, 0u, 0u);
    if (c8 == 0) lse[tok] = -INFINITY;
    return;
  }
  float tot = 0.f;
  for (int r = 0; r < n_rounds; ++r) tot += __expf(__ldg(lsepart + (int64_t)r * N + tok) - mx);
  const float LSE = mx + __logf(tot);
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  int r = 0;
  for (; r + 4 <= n_rounds; r += 4) {
    uint4 u[4];
    float wgt[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      u[k] = __ldg(reinterpret_cast<const uint4*>(opart + ((int64_t)(r + k) * N + tok) * kD + c8));
      const float l = __ldg(lsepart + (int64_t)(r + k) * N + tok);
      wgt[k] = (l == -INFINITY) ? 0.f : __expf(l - LSE);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float f[8];
      unpack8(u[k], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(wgt[k], f[i], acc[i]);
    }
  }
  for (; r < n_rounds; ++r) {
    const float l = __ldg(lsepart + (int64_t)r * N + tok);
    if (l == -INFINITY) continue;
    float f[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(opart + ((int64_t)r * N + tok) * kD + c8)), f);
    const float wgt = __expf(l - LSE);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = fmaf(wgt, f[i], acc[i]);
  }
  // per-round outputs pass through fp16: a value outside its range (or a
  // non-finite input) leaves a non-finite result, which is reported
  bool fin = isfinite(LSE);
#pragma unroll
  for (int i = 0; i < 8; ++i) fin = fin && isfinite(acc[i]);
  if (!fin) record_status(status, (int)LSH_ERR_RANGE);
  const uint4 hi = pack8_bf16(acc);
  *o16 = hi;
  if (out_lo) {
    float lo[8];
    const uint32_t w[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      lo[2 * i] = acc[2 * i] - __uint_as_float(w[i] << 16);
      lo[2 * i + 1] = acc[2 * i + 1] - __uint_as_float(w[i] & 0xffff0000u);
    }
    *reinterpret_cast<uint4*>(out_lo + tok * kD + c8) = pack8_bf16(lo);
  }
  if (c8 == 0) lse[tok] = LSE;
}

// D_i = dout_i . out_i; with init_grads also zero dqk and set dv = dout for
// self-attending rows, else 0.
template <typename T>
__global__ void __launch_bounds__(256)
bwd_prep_kernel(const T* __restrict__ out, const T* __restrict__ out_lo, const T* __restrict__ dout,
                const float* __restrict__ lse, float* __restrict__ D, float* __restrict__ dqk,
                float* __restrict__ dv, int64_t N, bool init_grads) {
  const int64_t tok = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 4;
  const int c4 = (threadIdx.x & 15) * 4;
  const bool live = tok < N;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f), g = o;
  if (live) {
    o = load4(out + tok * kD + c4);
    g = load4(dout + tok * kD + c4);
    if (out_lo) {
      float4 lo = load4(out_lo + tok * kD + c4);
      o.x += lo.x; o.y += lo.y; o.z += lo.z; o.w += lo.w;
    }
  }
  float d = warp_sum16(o.x * g.x + o.y * g.y + o.z * g.z + o.w * g.w);
  if (!live) return;
  if (c4 == 0) D[tok] = d;
  if (!init_grads) return;
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  store4(dqk + tok * kD + c4, z);
  store4(dv + tok * kD + c4, lse[tok] == -INFINITY ? g : z);
}

// Backward for one block of 64 query slots: recompute P from the final LSE,
// dS = P (dO.v - D); query-side dqk in registers, key-side dqk/dv by atomics.
template <typename T>
__global__ void __launch_bounds__(256)
bwd_round_kernel(const T* __restrict__ qk, const T* __restrict__ v, const T* __restrict__ dout,
                 const int32_t* __restrict__ perm, const float* __restrict__ lse,
                 const float* __restrict__ D, float* __restrict__ dqk, float* __restrict__ dv,
                 int L, int m, int n_rounds, int causal, float scale, float scale_log2,
                 int n_back, int n_fwd, int* status) {
  extern __shared__ float smem[];
  float(*Qs)[kP] = reinterpret_cast<float(*)[kP]>(smem);
  float(*Gs)[kP] = Qs + kQ;
  float(*Ks)[kP] = Gs + kQ;
  float(*Vs)[kP] = Ks + kK;
  float(*Ps)[kP] = Vs + kK;
  float(*Ss)[kP] = Ps + kQ;
  int* qpos = reinterpret_cast<int*>(Ss + kQ);
  int* kpos = qpos + kQ;
  float* qlse = reinterpret_cast<float*>(kpos + kK);
  float* qD = qlse + kQ;

  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int qblocks = L / kQ;
  const int qb = blockIdx.x % qblocks;
  const int64_t seg = blockIdx.x / qblocks;
  const int64_t bh = seg / n_rounds;
  const int32_t* pr = perm ? perm + seg * L : nullptr;
  const T* X = qk + bh * L * kD;
  const T* Vb = v + bh * L * kD;
  const T* Gb = dout + bh * L * kD;
  float* dX = dqk + bh * L * kD;
  float* dV = dv + bh * L * kD;
  const int t0 = qb * kQ, c = t0 / m;
  const int k_lo = (int)max((int64_t)0, (int64_t)(c - n_back) * m);
  const int k_hi = (int)min((int64_t)L, (int64_t)(c + 1 + n_fwd) * m);

  if (tid < kQ) {
    int q = checked_pos(pr, t0 + tid, L, status);
    qpos[tid] = q;
    qlse[tid] = lse[bh * L + q] * kLog2e;
    qD[tid] = D[bh * L + q];
  }
  __syncthreads();
  load_rows(Qs, X, qpos, tid);
  load_rows(Gs, Gb, qpos, tid);
  int myq[4];
  float ml[4], md[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) { myq[i] = qpos[ty * 4 + i]; ml[i] = qlse[ty * 4 + i]; md[i] = qD[ty * 4 + i]; }
  float dq[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) dq[i][j] = 0.f;

  for (int kt = k_lo; kt < k_hi; kt += kK) {
    __syncthreads();
    if (tid < kK) kpos[tid] = checked_pos(pr, kt + tid, L, status);
    __syncthreads();
    load_rows(Ks, X, kpos, tid);
    load_rows(Vs, Vb, kpos, tid);
    __syncthreads();
    float s[4][4], dp[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) { s[i][j] = 0.f; dp[i][j] = 0.f; }
#pragma unroll 4
    for (int k = 0; k < kD; ++k) {
      float a[4], g[4], b[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = Qs[ty * 4 + i][k]; g[i] = Gs[ty * 4 + i][k]; }
#pragma unroll
      for (int j = 0; j < 4; ++j) { b[j] = Ks[tx + 16 * j][k]; w[j] = Vs[tx + 16 * j][k]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          s[i][j] = fmaf(a[i], b[j], s[i][j]);
          dp[i][j] = fmaf(g[i], w[j], dp[i][j]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        int kp = kpos[tx + 16 * j];
        bool ok = (kp != myq[i]) && (!causal || kp < myq[i]) && (ml[i] != -INFINITY);
        float pv = ok ? exp2f(s[i][j] * scale_log2 - ml[i]) : 0.f;
        Ps[ty * 4 + i][tx + 16 * j] = pv;
        Ss[ty * 4 + i][tx + 16 * j] = pv * (dp[i][j] - md[i]);
      }
    __syncthreads();
    // query side: dq += dS K
#pragma unroll 4
    for (int k = 0; k < kK; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = Ss[ty * 4 + i][k];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Ks[k][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) dq[i][j] = fmaf(a[i], b[j], dq[i][j]);
    }
    // key side: dk = dS^T Q, dvv = P^T dO, for keys ty*4+i
    float dk[4][4], dvv[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) { dk[i][j] = 0.f; dvv[i][j] = 0.f; }
#pragma unroll 4
    for (int q = 0; q < kQ; ++q) {
      float sa[4], pa[4], qb4[4], gb4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { sa[i] = Ss[q][ty * 4 + i]; pa[i] = Ps[q][ty * 4 + i]; }
#pragma unroll
      for (int j = 0; j < 4; ++j) { qb4[j] = Qs[q][tx + 16 * j]; gb4[j] = Gs[q][tx + 16 * j]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          dk[i][j] = fmaf(sa[i], qb4[j], dk[i][j]);
          dvv[i][j] = fmaf(pa[i], gb4[j], dvv[i][j]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t krow = (int64_t)kpos[ty * 4 + i] * kD;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        atomicAdd(dX + krow + tx + 16 * j, scale * dk[i][j]);
        atomicAdd(dV + krow + tx + 16 * j, dvv[i][j]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t qrow = (int64_t)myq[i] * kD;
#pragma unroll
    for (int j = 0; j < 4; ++j) atomicAdd(dX + qrow + tx + 16 * j, scale * dq[i][j]);
  }
}

constexpr size_t kFwdSmem = (size_t)(2 * kQ + 2 * kK) * kP * 4 + (kQ + kK) * 4;
constexpr size_t kBwdSmem = (size_t)(4 * kQ + 2 * kK) * kP * 4 + (kQ + kK) * 4 + 2 * kQ * 4;

// fp16 copy of v for the tensor-core forward (exact inside the fp16 range;
// outside it a value becomes inf, which the combine's check reports).
__global__ void __launch_bounds__(256)
v_to_f16_kernel(const __nv_bfloat16* __restrict__ v, __half* __restrict__ v16, int64_t n8) {
  const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= n8) return;
  const uint4 w = __ldg(reinterpret_cast<const uint4*>(v) + k);
  reinterpret_cast<uint4*>(v16)[k] = make_uint4(tc_bf16x2_to_f16x2(w.x), tc_bf16x2_to_f16x2(w.y),
                                                tc_bf16x2_to_f16x2(w.z), tc_bf16x2_to_f16x2(w.w));
}

template <typename T>
cudaError_t fwd_t(const lsh_problem& p, const T* qk, const T* v, const int32_t* perm, T* out,
                  T* out_lo, float* lse, const FwdWs& ws, int* status, cudaStream_t s,
                  int n_back = 1, int n_fwd = 0, bool allow_tc = true) {
  const int64_t N = (int64_t)p.B * p.H * p.L;
  const int64_t blocks = (int64_t)p.B * p.H * p.n_rounds * (p.L / kQ);
  const unsigned cblocks = (unsigned)((N * 16 + 255) / 256);
  // the tensor-core forward reads an fp16 copy of v, kept in the unused half
  // of the per-round output buffer (sized for fp32, filled with fp16; N is
  // even, since L is a multiple of the chunk, so the copy ends inside it)
  __half* v16 = (__half*)((char*)ws.opart + align_up((size_t)p.n_rounds * N * kD * 2, 256));
  cudaError_t e = cudaErrorNotSupported;
  if (allow_tc && launch_attn_fwd_tc_ok(p)) {
    v_to_f16_kernel<<<(unsigned)((N * 8 + 255) / 256), 256, 0, s>>>(
        (const __nv_bfloat16*)v, v16, N * 8);
    note_launch();
    e = launch_attn_fwd_tc(p, qk, v16, perm, ws.opart, ws.lsepart, status, s);
  }
  if (e == cudaSuccess) {
    // the tensor-core forward handles bf16 problems only
    combine_f16_kernel<<<(unsigned)((N * 8 + 255) / 256), 256, 0, s>>>(
        (const __half*)ws.opart, ws.lsepart, (const __nv_bfloat16*)v, (__nv_bfloat16*)out,
        (__nv_bfloat16*)out_lo, lse, N, p.n_rounds, status);
    note_launch();
    return cudaGetLastError();
  }
  if (e != cudaErrorNotSupported) return e;
  e = cudaFuncSetAttribute(fwd_round_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kFwdSmem);
  if (e != cudaSuccess) return e;
  fwd_round_kernel<T><<<(unsigned)blocks, 256, kFwdSmem, s>>>(
      qk, v, perm, ws.opart, ws.lsepart, p.L, p.chunk, p.n_rounds, N, p.causal,
      p.scale * kLog2e, n_back, n_fwd, status);
  combine_kernel<T, float><<<cblocks, 256, 0, s>>>(ws.opart, ws.lsepart, v, out, out_lo, lse, N,
                                                   p.n_rounds);
  note_launch(2);
  return cudaGetLastError();
}

template <typename T>
cudaError_t bwd_t(const lsh_problem& p, const T* qk, const T* v, const int32_t* perm, const T* out,
                  const T* out_lo, const float* lse, const T* dout, float* dqk, float* dv, float* D, int* status,
                  cudaStream_t s, int n_back = 1, int n_fwd = 0, bool allow_tc = true) {
  const int64_t N = (int64_t)p.B * p.H * p.L;
  const int64_t blocks = (int64_t)p.B * p.H * p.n_rounds * (p.L / kQ);
  cudaError_t e = cudaFuncSetAttribute(bwd_round_kernel<T>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBwdSmem);
  if (e != cudaSuccess) return e;
  if (allow_tc && bwd_tc_ws_bytes(p) > 0) {
    e = launch_attn_bwd_tc(p, qk, v, dout, out, out_lo, perm, lse, D, dqk, dv,
                           (char*)D + align_up((size_t)N * 4, 256), status, s);
    return e == cudaSuccess ? cudaGetLastError() : e;
  }
  bwd_prep_kernel<T><<<(unsigned)((N * 16 + 255) / 256), 256, 0, s>>>(out, out_lo, dout, lse, D, dqk, dv,
                                                                        N, true);
  note_launch();
  bwd_round_kernel<T><<<(unsigned)blocks, 256, kBwdSmem, s>>>(
      qk, v, dout, perm, lse, D, dqk, dv, p.L, p.chunk, p.n_rounds, p.causal, p.scale,
      p.scale * kLog2e, n_back, n_fwd, status);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

// ---- local attention: the same kernels in the identity order ------------
namespace {

__global__ void iota_kernel(int32_t* __restrict__ perm, int L, int64_t total) {
  const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (k < total) perm[k] = (int32_t)(k % L);
}

// Look-back 1 and no look-ahead is the LSH window: bf16 problems with chunk
// 64 take the tensor-core kernels with an identity permutation.
bool local_tc(const lsh_problem& p, int n_back, int n_fwd) {
  return p.dtype == LSH_BF16 && p.chunk == 64 && n_back == 1 && n_fwd == 0 && p.scale > 0.f;
}

int32_t* fill_identity(const lsh_problem& p, void* at, cudaStream_t s) {
  const int64_t total = (int64_t)p.B * p.H * p.L;
  int32_t* perm = (int32_t*)at;
  iota_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(perm, p.L, total);
  note_launch();
  return perm;
}

}  // namespace

size_t local_fwd_ws_bytes(const lsh_problem& p, int n_back, int n_fwd) {
  const size_t N = (size_t)p.B * p.H * p.L;
  return fwd_ws_bytes(p) + (local_tc(p, n_back, n_fwd) ? align_up(N * 4, 256) : 0);
}

cudaError_t launch_local_fwd(const lsh_problem& p, int n_back, int n_fwd, const void* qk,
                             const void* v, void* out, void* out_lo, float* lse, void* ws,
                             int* status, cudaStream_t s) {
  const FwdWs w = fwd_ws_carve(p, ws);
  if (local_tc(p, n_back, n_fwd)) {
    const int32_t* perm = fill_identity(p, (char*)ws + fwd_ws_bytes(p), s);
    return fwd_t(p, (const __nv_bfloat16*)qk, (const __nv_bfloat16*)v, perm, (__nv_bfloat16*)out,
                 (__nv_bfloat16*)out_lo, lse, w, status, s);
  }
  if (p.dtype == LSH_BF16)
    return fwd_t(p, (const __nv_bfloat16*)qk, (const __nv_bfloat16*)v, (const int32_t*)nullptr,
                 (__nv_bfloat16*)out, (__nv_bfloat16*)out_lo, lse, w, status, s, n_back, n_fwd,
                 false);
  return fwd_t(p, (const float*)qk, (const float*)v, (const int32_t*)nullptr, (float*)out,
               (float*)nullptr, lse, w, status, s, n_back, n_fwd, false);
}

size_t local_bwd_ws_bytes(const lsh_problem& p, int n_back, int n_fwd) {
  const size_t N = (size_t)p.B * p.H * p.L;
  if (local_tc(p, n_back, n_fwd)) return bwd_ws_bytes(p) + align_up(N * 4, 256);
  return align_up(N * 4, 256);
}

cudaError_t launch_local_bwd(const lsh_problem& p, int n_back, int n_fwd, const void* qk,
                             const void* v, const void* out, const void* out_lo, const float* lse,
                             const void* dout, float* dqk, float* dv, void* ws, int* status,
                             cudaStream_t s) {
  float* D = (float*)ws;
  if (local_tc(p, n_back, n_fwd)) {
    const int32_t* perm = fill_identity(p, (char*)ws + bwd_ws_bytes(p), s);
    return bwd_t(p, (const __nv_bfloat16*)qk, (const __nv_bfloat16*)v, perm,
                 (const __nv_bfloat16*)out, (const __nv_bfloat16*)out_lo, lse,
                 (const __nv_bfloat16*)dout, dqk, dv, D, status, s);
  }
  if (p.dtype == LSH_BF16)
    return bwd_t(p, (const __nv_bfloat16*)qk, (const __nv_bfloat16*)v, (const int32_t*)nullptr,
                 (const __nv_bfloat16*)out, (const __nv_bfloat16*)out_lo, lse,
                 (const __nv_bfloat16*)dout, dqk, dv, D, status, s, n_back, n_fwd, false);
  return bwd_t(p, (const float*)qk, (const float*)v, (const int32_t*)nullptr, (const float*)out,
               (const float*)nullptr, lse, (const float*)dout, dqk, dv, D, status, s, n_back, n_fwd,
               false);
}

size_t fwd_ws_bytes(const lsh_problem& p) {
  const size_t N = (size_t)p.B * p.H * p.L;
  return align_up((size_t)p.n_rounds * N * kD * 4, 256) + align_up((size_t)p.n_rounds * N * 4, 256);
}

FwdWs fwd_ws_carve(const lsh_problem& p, void* ws) {
  const size_t N = (size_t)p.B * p.H * p.L;
  FwdWs w;
  w.opart = (float*)ws;
  w.lsepart = (float*)((char*)ws + align_up((size_t)p.n_rounds * N * kD * 4, 256));
  return w;
}

cudaError_t launch_attn_fwd(const lsh_problem& p, const void* qk, const void* v,
                            const int32_t* perm, void* out, void* out_lo, float* lse,
                            const FwdWs& ws, int* status, cudaStream_t s) {
  if (p.dtype == LSH_BF16)
    return fwd_t(p, (const __nv_bfloat16*)qk, (const __nv_bfloat16*)v, perm, (__nv_bfloat16*)out,
                 (__nv_bfloat16*)out_lo, lse, ws, status, s);
  return fwd_t(p, (const float*)qk, (const float*)v, perm, (float*)out, (float*)nullptr, lse, ws,
               status, s);
}

size_t bwd_ws_bytes(const lsh_problem& p) {
  return align_up((size_t)p.B * p.H * p.L * 4, 256) + bwd_tc_ws_bytes(p);
}

cudaError_t launch_attn_bwd(const lsh_problem& p, const void* qk, const void* v,
                            const int32_t* perm, const void* out, const void* out_lo,
                            const float* lse, const void* dout, float* dqk, float* dv, void* ws,
                            int* status, cudaStream_t s) {
  float* D = (float*)ws;
  if (p.dtype == LSH_BF16)
    return bwd_t(p, (const __nv_bfloat16*)qk, (const __nv_bfloat16*)v, perm,
                 (const __nv_bfloat16*)out, (const __nv_bfloat16*)out_lo, lse,
                 (const __nv_bfloat16*)dout, dqk, dv, D, status, s);
  return bwd_t(p, (const float*)qk, (const float*)v, perm, (const float*)out,
               (const float*)nullptr, lse, (const float*)dout, dqk, dv, D, status, s);
}

}  // namespace lsh
