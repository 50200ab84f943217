// Per-round chunk attention on the 5th-generation tensor cores (bf16 inputs,
// chunk m = 64, head size 64).
//
// "Reformer: The Efficient Transformer" (research.elamur.ai summary page),
// Key points "LSH attention" (each chunk of m sorted positions attends to
// itself and the chunk before it) and "Shared-QK Transformer" (keys are the
// queries; no attending to oneself unless nothing else is valid).
//
// One MMA tile covers a PAIR of query chunks (2p, 2p+1): M = 128 queries
// against the 192 keys of chunks 2p-1, 2p, 2p+1. Rows of chunk 2p use key
// blocks 0-1, rows of chunk 2p+1 use blocks 1-2; the unused block of each
// row gets P = 0. Queries and keys are the same rows (shared QK), so a chunk
// is gathered once and serves as query tile, key tile and value tile.
//
// Warp roles (persistent CTA, one per SM, walking units of kUnit pairs of one
// (batch, head, round) segment):
//   warps 0-3 : gather rows of x and v through perm (16-byte loads), convert
//               bf16 -> fp16 (exact for |values| < 65504), store them in the
//               128-byte-swizzled K-major layout into a 4-slot ring; chunk
//               2p0-1 of a unit's first pair goes to a separate buffer;
//   warp 4    : TMEM allocation; one thread issues S = Q K^T (3 MMAs of
//               128x64x64 per pair into a double-buffered TMEM S) and
//               O = P V (P from shared memory, V as the MN-major operand);
//   warps 5-8 : softmax, one query row per thread: S from TMEM, masks
//               (causal / self), row max, exp2, row sum, P (fp16) into shared
//               memory; then O from TMEM, scaled by 1/l, written as the fp16
//               per-round output in original token order with lse_r.
// fp16 operands for P V keep P's rounding error at 2^-11 (bf16 would add
// about 3e-3 to O on the 64K workload).
#include <cuda_fp16.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"
#include "tma_host.h"

namespace lsh {
namespace {

using namespace tc;

constexpr int kM = 64;            // chunk
constexpr int kUnit = 8;          // pairs per work unit
constexpr int kSlots = 4;         // pair slots in the ring
constexpr int kTile = 64 * 128;   // one chunk of 64 rows x 64 fp16 = 8 KB
constexpr int kSlotBytes = 4 * kTile;   // x_even | x_odd | v_even | v_odd
constexpr int kPreBytes = 2 * kTile;    // x_prev | v_prev
constexpr int kPBytes = 3 * 128 * 128;  // P: 3 blocks of 128 rows x 64 fp16
constexpr int kThreads = 288;
constexpr uint32_t kSCols = 192;

struct __align__(8) FwdBar {
  uint64_t slot_full[kSlots];
  uint64_t slot_free[kSlots];
  uint64_t pre_free;
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t p_full;
  uint64_t p_free;
  uint64_t o_free[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  int kpos[kSlots][128];   // original positions of the slot's even|odd rows
  int kpos_pre[64];
};

constexpr size_t kSmemBytes = 1024 + kSlots * kSlotBytes + kPreBytes + kPBytes + sizeof(FwdBar);

struct Job {
  int64_t seg;   // (b*H + h)*n_rounds + r
  int p;         // pair index within the segment
  bool first;    // first pair of its unit (its previous chunk is gathered separately)
};

// Walks the CTA's units in order; every role iterates the same sequence.
struct JobIter {
  int64_t unit, n_units, stride;
  int units_per_seg, n_pairs, k;
  __device__ JobIter(int64_t u0, int64_t nu, int64_t st, int ups, int np)
      : unit(u0), n_units(nu), stride(st), units_per_seg(ups), n_pairs(np), k(0) {}
  __device__ bool next(Job& j) {
    while (unit < n_units) {
      const int64_t seg = unit / units_per_seg;
      const int p0 = (int)(unit % units_per_seg) * kUnit;
      const int p = p0 + k;
      if (k < kUnit && p < n_pairs) {
        j.seg = seg;
        j.p = p;
        j.first = (k == 0);
        ++k;
        return true;
      }
      unit += stride;
      k = 0;
    }
    return false;
  }
};

// 2^x with the hardware approximation (relative error about 2^-22; -inf -> 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t cvt_bf16x2_to_f16x2(uint32_t u) {
  const float lo = __uint_as_float(u << 16), hi = __uint_as_float(u & 0xffff0000u);
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Gathers the 64 rows of chunk c of segment `seg` (x and v), converting to fp16
// and storing swizzled. Thread t: row t>>1, 16-byte chunks 4*(t&1)..+3.
__device__ __forceinline__ void gather_chunk(const __nv_bfloat16* __restrict__ qk,
                                             const __nv_bfloat16* __restrict__ v,
                                             const int32_t* __restrict__ perm, int64_t seg,
                                             int64_t bh, int L, int c, uint8_t* x_dst,
                                             uint8_t* v_dst, int* kpos, int t, int* status) {
  const int row = t >> 1, half = t & 1;
  int pos = perm[seg * L + (int64_t)c * kM + row];
  if ((unsigned)pos >= (unsigned)L) {
    if (status) atomicExch(status, (int)LSH_ERR_DEVICE_CHECK);
    pos = 0;
  }
  if (half == 0) kpos[row] = pos;
  const uint4* xs = reinterpret_cast<const uint4*>(qk + (bh * L + pos) * 64) + half * 4;
  const uint4* vs = reinterpret_cast<const uint4*>(v + (bh * L + pos) * 64) + half * 4;
  uint4 xv[4], vv[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    xv[i] = __ldg(xs + i);
    vv[i] = __ldg(vs + i);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int ch = half * 4 + i;
    const uint32_t off = row * 128 + ((ch ^ (row & 7)) << 4);
    uint4 a, b;
    a.x = cvt_bf16x2_to_f16x2(xv[i].x); a.y = cvt_bf16x2_to_f16x2(xv[i].y);
    a.z = cvt_bf16x2_to_f16x2(xv[i].z); a.w = cvt_bf16x2_to_f16x2(xv[i].w);
    b.x = cvt_bf16x2_to_f16x2(vv[i].x); b.y = cvt_bf16x2_to_f16x2(vv[i].y);
    b.z = cvt_bf16x2_to_f16x2(vv[i].z); b.w = cvt_bf16x2_to_f16x2(vv[i].w);
    *reinterpret_cast<uint4*>(x_dst + off) = a;
    *reinterpret_cast<uint4*>(v_dst + off) = b;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_tc_kernel(const __nv_bfloat16* __restrict__ qk, const __nv_bfloat16* __restrict__ v,
                   const int32_t* __restrict__ perm, __half* __restrict__ opart,
                   float* __restrict__ lsepart, int L, int n_rounds, int64_t N, int causal,
                   float scale_log2, int64_t n_units, int units_per_seg, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* slots = smem;
  uint8_t* pre = slots + kSlots * kSlotBytes;
  uint8_t* pbuf = pre + kPreBytes;
  FwdBar* bar = (FwdBar*)(pbuf + kPBytes);
  volatile int* abort = &bar->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_chunks = L / kM;
  const int n_pairs = (n_chunks + 1) / 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&bar->slot_full[s], 128);
      mbar_init(&bar->slot_free[s], 1);
    }
    mbar_init(&bar->pre_free, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar->s_full[b], 1);
      mbar_init(&bar->s_free[b], 128);
      mbar_init(&bar->o_free[b], 128);
    }
    mbar_init(&bar->p_full, 128);
    mbar_init(&bar->p_free, 1);
    mbar_init(&bar->mma_done, 1);
    bar->abort = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(&bar->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp < 4) {
    // ------------------------------------------------ producers
    const int t = threadIdx.x;
    JobIter it(blockIdx.x, n_units, gridDim.x, units_per_seg, n_pairs);
    Job j;
    int n = 0, pre_uses = 0;
    while (it.next(j)) {
      const int s = n % kSlots;
      if (n >= kSlots &&
          !mbar_wait(&bar->slot_free[s], (uint32_t)(n / kSlots - 1) & 1u, abort, status))
        break;
      const int64_t bh = j.seg / n_rounds;
      uint8_t* sl = slots + s * kSlotBytes;
      const int ce = 2 * j.p, co = 2 * j.p + 1;
      if (j.first && j.p > 0) {
        if (pre_uses > 0 &&
            !mbar_wait(&bar->pre_free, (uint32_t)(pre_uses - 1) & 1u, abort, status))
          break;
        gather_chunk(qk, v, perm, j.seg, bh, L, ce - 1, pre, pre + kTile, bar->kpos_pre, t, status);
        ++pre_uses;
      }
      gather_chunk(qk, v, perm, j.seg, bh, L, ce, sl, sl + 2 * kTile, bar->kpos[s], t, status);
      if (co < n_chunks)
        gather_chunk(qk, v, perm, j.seg, bh, L, co, sl + kTile, sl + 3 * kTile, bar->kpos[s] + 64,
                     t, status);
      fence_proxy_async();
      mbar_arrive(&bar->slot_full[s]);
      ++n;
    }
  } else if (warp == 4) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_f16(128, 64, 0, false, false);   // Q K^T, both K-major
      const uint32_t idesc_o = idesc_f16(128, 64, 0, false, true);    // P V, V MN-major
      const uint32_t slots_a = smem_u32(slots), pre_a = smem_u32(pre), p_a = smem_u32(pbuf);
      JobIter it(blockIdx.x, n_units, gridDim.x, units_per_seg, n_pairs);
      Job cur, nxt;
      bool have_cur = it.next(cur);
      int n = 0;
      bool ok = true;
      // issue S for job n (slot n%kSlots, buffer n&1)
      auto issue_s = [&](const Job& jb, int nn) -> bool {
        const int s = nn % kSlots, b = nn & 1;
        if (!mbar_wait(&bar->slot_full[s], (uint32_t)(nn / kSlots) & 1u, abort, status)) return false;
        if (nn >= 2 && !mbar_wait(&bar->s_free[b], (uint32_t)(nn / 2 - 1) & 1u, abort, status))
          return false;
        tc_fence_after();
        const uint32_t sl = slots_a + s * kSlotBytes;
        const uint32_t d = tmem + (uint32_t)b * kSCols;
        const bool has_prev = jb.p > 0, has_odd = 2 * jb.p + 1 < n_chunks;
        const uint32_t prev_x =
            jb.first ? pre_a : slots_a + ((nn + kSlots - 1) % kSlots) * kSlotBytes + kTile;
        const uint32_t keys[3] = {prev_x, sl, sl + kTile};
        for (int kb = 0; kb < 3; ++kb) {
          if ((kb == 0 && !has_prev) || (kb == 2 && !has_odd)) continue;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t a = smem_desc(sl + ks * 32, 16, 1024);
            const uint64_t bd = smem_desc(keys[kb] + ks * 32, 16, 1024);
            mma_ss(d + kb * 64, a, bd, idesc_s, ks > 0 ? 1u : 0u);
          }
        }
        mma_commit(&bar->s_full[b]);
        return true;
      };
      if (have_cur) ok = issue_s(cur, 0);
      while (have_cur && ok) {
        const bool have_nxt = it.next(nxt);
        if (have_nxt && !issue_s(nxt, n + 1)) break;
        // O = P V for job n
        if (!mbar_wait(&bar->p_full, (uint32_t)n & 1u, abort, status)) break;
        if (n >= 2 && !mbar_wait(&bar->o_free[n & 1], (uint32_t)(n / 2 - 1) & 1u, abort, status))
          break;
        tc_fence_after();
        const int s = n % kSlots;
        const uint32_t sl = slots_a + s * kSlotBytes;
        const bool has_prev = cur.p > 0, has_odd = 2 * cur.p + 1 < n_chunks;
        const uint32_t prev_v = cur.first
                                    ? pre_a + kTile
                                    : slots_a + ((n + kSlots - 1) % kSlots) * kSlotBytes + 3 * kTile;
        const uint32_t vals[3] = {prev_v, sl + 2 * kTile, sl + 3 * kTile};
        const uint32_t d = tmem + 2 * kSCols + (uint32_t)(n & 1) * 64;
        bool acc = false;
        for (int kb = 0; kb < 3; ++kb) {
          if ((kb == 0 && !has_prev) || (kb == 2 && !has_odd)) continue;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t a = smem_desc(p_a + kb * (128 * 128) + ks * 32, 16, 1024);
            const uint64_t bd = smem_desc(vals[kb] + ks * 2048, 8192, 1024);
            mma_ss(d, a, bd, idesc_o, acc ? 1u : 0u);
            acc = true;
          }
        }
        mma_commit(&bar->p_free);                       // P consumed, O(n) ready
        if (n >= 1) mma_commit(&bar->slot_free[(n - 1) % kSlots]);
        if (cur.first && cur.p > 0) mma_commit(&bar->pre_free);
        cur = nxt;
        have_cur = have_nxt;
        ++n;
      }
      mma_commit(&bar->mma_done);
      int dummy = 0;
      mbar_wait(&bar->mma_done, 0, (volatile int*)&dummy, status);
    }
  } else {
    // ------------------------------------------------ softmax + epilogue
    const int q = warp & 3;                     // TMEM lane quarter (rows 32q..32q+31)
    const int row = q * 32 + lane;              // query row in the pair tile
    const bool odd_row = row >= 64;             // row belongs to chunk 2p+1
    const int kb0 = odd_row ? 1 : 0;            // first key block of this row
    JobIter it(blockIdx.x, n_units, gridDim.x, units_per_seg, n_pairs);
    Job j;
    int n = 0;
    // pending epilogue state of the previous job
    bool pend = false, pend_write = false;
    float pend_inv_l = 0.f, pend_lse = 0.f;
    int64_t pend_row = 0;
    auto epilogue = [&](int nn) {
      // O(nn) is complete (p_free phase nn observed by the caller)
      tc_fence_after();
      const uint32_t taddr =
          tmem + ((uint32_t)(q * 32) << 16) + 2 * kSCols + (uint32_t)(nn & 1) * 64;
      uint32_t o0[32], o1[32];
      tmem_ld32(taddr, o0);
      tmem_ld32(taddr + 32, o1);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bar->o_free[nn & 1]);
      if (pend_write) {
        uint4* dst = reinterpret_cast<uint4*>(opart + pend_row * 64);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 w;
          __half2 h0 = __floats2half2_rn(__uint_as_float(o0[8 * c + 0]) * pend_inv_l,
                                         __uint_as_float(o0[8 * c + 1]) * pend_inv_l);
          __half2 h1 = __floats2half2_rn(__uint_as_float(o0[8 * c + 2]) * pend_inv_l,
                                         __uint_as_float(o0[8 * c + 3]) * pend_inv_l);
          __half2 h2 = __floats2half2_rn(__uint_as_float(o0[8 * c + 4]) * pend_inv_l,
                                         __uint_as_float(o0[8 * c + 5]) * pend_inv_l);
          __half2 h3 = __floats2half2_rn(__uint_as_float(o0[8 * c + 6]) * pend_inv_l,
                                         __uint_as_float(o0[8 * c + 7]) * pend_inv_l);
          w.x = *reinterpret_cast<uint32_t*>(&h0); w.y = *reinterpret_cast<uint32_t*>(&h1);
          w.z = *reinterpret_cast<uint32_t*>(&h2); w.w = *reinterpret_cast<uint32_t*>(&h3);
          dst[c] = w;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 w;
          __half2 h0 = __floats2half2_rn(__uint_as_float(o1[8 * c + 0]) * pend_inv_l,
                                         __uint_as_float(o1[8 * c + 1]) * pend_inv_l);
          __half2 h1 = __floats2half2_rn(__uint_as_float(o1[8 * c + 2]) * pend_inv_l,
                                         __uint_as_float(o1[8 * c + 3]) * pend_inv_l);
          __half2 h2 = __floats2half2_rn(__uint_as_float(o1[8 * c + 4]) * pend_inv_l,
                                         __uint_as_float(o1[8 * c + 5]) * pend_inv_l);
          __half2 h3 = __floats2half2_rn(__uint_as_float(o1[8 * c + 6]) * pend_inv_l,
                                         __uint_as_float(o1[8 * c + 7]) * pend_inv_l);
          w.x = *reinterpret_cast<uint32_t*>(&h0); w.y = *reinterpret_cast<uint32_t*>(&h1);
          w.z = *reinterpret_cast<uint32_t*>(&h2); w.w = *reinterpret_cast<uint32_t*>(&h3);
          dst[4 + c] = w;
        }
        lsepart[pend_row] = pend_lse;
      }
    };
    bool ok = true;
    while (ok && it.next(j)) {
      const int b = n & 1, s = n % kSlots;
      if (!mbar_wait(&bar->s_full[b], (uint32_t)(n / 2) & 1u, abort, status)) break;
      tc_fence_after();
      // S row: 128 columns starting at key block kb0
      uint32_t sv[128];
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)b * kSCols + kb0 * 64;
      tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      tmem_ld32(taddr + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
      tmem_ld32(taddr + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bar->s_free[b]);
      const bool has_prev = j.p > 0, has_odd = 2 * j.p + 1 < n_chunks;
      const bool row_live = !odd_row || has_odd;
      const int qpos = bar->kpos[s][row];
      const int* kp_lo = (kb0 == 0) ? (j.first ? bar->kpos_pre
                                               : bar->kpos[(n + kSlots - 1) % kSlots] + 64)
                                    : bar->kpos[s];
      const int* kp_hi = (kb0 == 0) ? bar->kpos[s] : bar->kpos[s] + 64;
      const bool lo_ok = (kb0 == 0) ? has_prev : true;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        const int kp = (c < 64) ? kp_lo[c] : kp_hi[c - 64];
        const bool blk_ok = (c < 64) ? lo_ok : true;
        const bool valid = blk_ok && (causal ? (kp < qpos) : (kp != qpos));
        const float x = valid ? __uint_as_float(sv[c]) * scale_log2 : -INFINITY;
        sv[c] = __float_as_uint(x);
        mx = fmaxf(mx, x);
      }
      const float ms = (mx == -INFINITY) ? 0.f : mx;
      // P buffer is free once PV(n-1) is done; that also completes O(n-1)
      if (n >= 1 && !mbar_wait(&bar->p_free, (uint32_t)(n - 1) & 1u, abort, status)) break;
      // P row: key blocks kb0 and kb0+1 hold exp2(s - max), the third block is 0
      float l = 0.f;
      uint8_t* prow = pbuf + row * 128;
      const uint32_t sw = (uint32_t)(row & 7);
#pragma unroll
      for (int g = 0; g < 16; ++g) {             // 16 groups of 8 columns
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float e0 = ex2(__uint_as_float(sv[8 * g + 2 * e]) - ms);
          const float e1 = ex2(__uint_as_float(sv[8 * g + 2 * e + 1]) - ms);
          l += e0 + e1;
          __half2 h = __floats2half2_rn(e0, e1);
          w[e] = *reinterpret_cast<uint32_t*>(&h);
        }
        const int blk = kb0 + (g >> 3), ch = g & 7;
        *reinterpret_cast<uint4*>(prow + blk * (128 * 128) + (((uint32_t)ch ^ sw) << 4)) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
      {
        const int zblk = odd_row ? 0 : 2;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          *reinterpret_cast<uint4*>(prow + zblk * (128 * 128) + (((uint32_t)ch ^ sw) << 4)) =
              make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async();
      mbar_arrive(&bar->p_full);
      if (pend) epilogue(n - 1);
      pend = true;
      pend_write = row_live;
      const int64_t bh = j.seg / n_rounds;
      const int r = (int)(j.seg % n_rounds);
      pend_row = (int64_t)r * N + bh * L + qpos;
      const bool has = mx != -INFINITY;
      pend_inv_l = has ? 1.f / l : 0.f;
      pend_lse = has ? (mx + log2f(l)) * kLn2 : -INFINITY;
      ++n;
    }
    if (ok && pend && !*abort) {
      if (mbar_wait(&bar->p_free, (uint32_t)(n - 1) & 1u, abort, status)) epilogue(n - 1);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

size_t fwd_tc_partial_bytes(const lsh_problem& p) {
  return (size_t)p.n_rounds * p.B * p.H * p.L * 64 * sizeof(__half);
}

cudaError_t launch_attn_fwd_tc(const lsh_problem& p, const void* qk, const void* v,
                               const int32_t* perm, void* opart_f16, float* lsepart, int* status,
                               cudaStream_t s) {
  if (p.dtype != LSH_BF16 || p.chunk != kM) return cudaErrorNotSupported;
  const int n_chunks = p.L / kM;
  const int n_pairs = (n_chunks + 1) / 2;
  const int units_per_seg = (n_pairs + kUnit - 1) / kUnit;
  const int64_t n_segs = (int64_t)p.B * p.H * p.n_rounds;
  const int64_t n_units = n_segs * units_per_seg;
  const int64_t N = (int64_t)p.B * p.H * p.L;
  int grid = sm_count();
  if ((int64_t)grid > n_units) grid = (int)n_units;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  attn_fwd_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(
      (const __nv_bfloat16*)qk, (const __nv_bfloat16*)v, perm, (__half*)opart_f16, lsepart, p.L,
      p.n_rounds, N, p.causal, p.scale * kLog2e, n_units, units_per_seg, status);
  note_launch();
  return cudaGetLastError();
}

}  // namespace lsh
