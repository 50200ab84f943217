// Backward pass of chunked LSH attention on the 5th-generation tensor cores
// (bf16 inputs, chunk m = 64, head size 64), recomputing the attention
// weights instead of storing them ("Reformer: The Efficient Transformer",
// research.elamur.ai summary page, Summary: activations are recomputed).
//
// With the final log-sum-exp LSE_i of each query and D_i = dout_i . O_i:
//   P_ij = exp(s_ij - LSE_i),  dS_ij = P_ij (dout_i . v_j - D_i),
//   dv_j += P_ij dout_i,  dqk_j += scale dS_ij x_i (key side),
//   dqk_i += scale dS_ij x_j (query side: keys are the queries).
//
// Work item: a PAIR of key chunks (2p, 2p+1) of one (batch, head, round)
// segment — 128 keys. The queries that see them are chunks 2p, 2p+1, 2p+2
// (chunk c sees chunks c-1 and c), 192 queries in three blocks; key rows of
// chunk 2p use query blocks 0-1, rows of chunk 2p+1 use blocks 1-2.
//   S^T  = X_K X_Q^T  and  dP^T = V_K dO_Q^T       (M=128 keys, N=3x64)
//   P^T, dS^T per key row (one thread per TMEM lane)
//   dV   = P^T dO_Q   (P^T from TMEM)              (complete for the keys)
//   dK   = dS^T X_Q   (dS^T from shared memory)    (complete for the keys)
//   R0   = dS[blocks 0,1] X_K  — the query-side term for chunks 2p, 2p+1,
//          i.e. for the same tokens as the key rows, lane for lane;
//   R1   = dS[block 2, zeros] X_K — the query-side term for chunk 2p+2
//          (its other half comes from the next pair's work item).
// The dS operands of R0/R1 are the transposed (MN-major) reading of the
// dS^T tile. Each key row then adds scale*(dK + R0) to dqk and dV to dv with
// vector atomics (rounds and neighbouring items accumulate there); rows of
// chunk 2p+2 add scale*R1.
//
// Warp roles (persistent CTA, one per SM):
//   warps 0-3: producers — cp.async gathers of x, dout (3 chunks) and v (2
//              chunks) into a 2-slot ring, in-place bf16 -> fp16 conversion,
//              per-query position, log2-scaled LSE and D;
//   warp 4   : TMEM allocation and the MMA-issuing thread;
//   warps 5-8 and 9-12: two warpgroups, one thread per key row in each; the
//              first takes the row's first query block, the second its second
//              (P and dS are elementwise once LSE and D are known, so the two
//              halves need no exchange); then the gradient epilogue with
//              atomics, dV and R1 from the first warpgroup, dK + R0 from the
//              second.
#include <cuda_fp16.h>
#include <stddef.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"
#include "tma_host.h"

namespace lsh {
namespace {

using namespace tc;

constexpr int kM = 64;
constexpr int kUnit = 8;
constexpr int kSlots = 2;
constexpr int kTile = 64 * 128;        // 64 rows x 64 16-bit values
// slot: x0 x1 x2 | v0 v1 | d0 d1 d2
constexpr int kX = 0, kV = 3 * kTile, kDo = 5 * kTile;
constexpr int kSlotBytes = 8 * kTile;  // 64 KB
constexpr int kDsBlock = 128 * 128;    // 128 key rows x 64 query columns
constexpr int kDsBytes = 4 * kDsBlock; // dS^T blocks 0,1,2 + a zero block
constexpr int kThreads = 416;
// TMEM columns
constexpr uint32_t kColS = 0, kColDp = 192;      // S^T, dP^T
constexpr uint32_t kColDv = 96, kColDk = 288;    // accumulators in their upper halves
constexpr uint32_t kColR0 = 384, kColR1 = 448;
// P^T (fp16 pairs, 3 x 32 columns) lives in the R0/R1 columns while they are
// idle: written after the previous item's flush, read by the dV MMAs, which
// run before the R0/R1 MMAs that overwrite it (MMAs complete in issue order).
// The S^T/dP^T columns are read by both key-row warpgroups, so nothing is
// written there before both have read them.
constexpr uint32_t kColP = 384;

struct __align__(16) BwdBar {
  uint64_t slot_full[kSlots];
  uint64_t slot_free[kSlots];
  uint64_t s_full;
  uint64_t p_full;
  uint64_t g_full;
  uint64_t g_free;
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  alignas(16) int qpos[kSlots][192];     // positions of query columns (= key rows for 0..127)
  alignas(16) float lse2[kSlots][192];   // LSE * log2(e); +inf for self-attending rows
  alignas(16) float dval[kSlots][192];   // D = dout . out
};
static_assert(offsetof(BwdBar, qpos) % 16 == 0 && offsetof(BwdBar, lse2) % 16 == 0 &&
                  offsetof(BwdBar, dval) % 16 == 0,
              "per-column arrays are read with 16-byte loads");

constexpr size_t kSmemBytes = 1024 + kSlots * kSlotBytes + kDsBytes + sizeof(BwdBar);

struct Job {
  int64_t seg;
  int p;
  bool first, last;   // first / last pair of its unit
};

struct JobIter {
  int unit, n_units, stride;
  int units_per_seg, n_pairs, k;
  __device__ JobIter(int u0, int nu, int st, int ups, int np)
      : unit(u0), n_units(nu), stride(st), units_per_seg(ups), n_pairs(np), k(0) {}
  __device__ bool next(Job& j) {
    while (unit < n_units) {
      const int seg = unit / units_per_seg;
      const int p0 = (unit - seg * units_per_seg) * kUnit;
      const int p = p0 + k;
      if (k < kUnit && p < n_pairs) {
        j.seg = seg;
        j.p = p;
        j.first = (k == 0);
        j.last = (k == kUnit - 1) || (p + 1 == n_pairs);
        ++k;
        return true;
      }
      unit += stride;
      k = 0;
    }
    return false;
  }
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

__device__ __forceinline__ void issue_row(const __nv_bfloat16* __restrict__ src_row, uint8_t* tile,
                                          int row, int half) {
  const uint32_t base = smem_u32(tile) + row * 128;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int ch = half * 4 + i;
    cp_async16(base + (((uint32_t)ch ^ (uint32_t)(row & 7)) << 4), src_row + ch * 8);
  }
}
__device__ __forceinline__ void convert_row(uint8_t* tile, int row, int half) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int ch = half * 4 + i;
    convert_piece_bf16_to_f16(tile + row * 128 + ((ch ^ (row & 7)) << 4));
  }
}

// Adds scale * (64 consecutive TMEM columns of each lane [+ another 64]) to
// the 64-float global row `row_of_lane` of that lane (token `tok`, or none
// when tok < 0). The warp stages its 32 half-rows in shared memory and
// re-reads them so that each vector atomic instruction covers four whole
// 128-byte lines (8 lanes per row) instead of 32 scattered 16-byte pieces.
constexpr int kStageStride = 144;   // bytes per staged half-row (128 + 16 pad)
__device__ __forceinline__ void flush_rows(float* base, int tok, uint32_t ta, uint32_t tb,
                                           bool two, float scale, uint8_t* stage, int lane) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t a[32], b[32];
    tmem_ld32(ta + 32 * h, a);
    if (two) tmem_ld32(tb + 32 * h, b);
    tmem_ld_wait();
    uint8_t* mine = stage + lane * kStageStride;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float x[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float val = __uint_as_float(a[4 * c + e]);
        if (two) val += __uint_as_float(b[4 * c + e]);
        x[e] = val * scale;
      }
      *reinterpret_cast<float4*>(mine + 16 * c) = make_float4(x[0], x[1], x[2], x[3]);
    }
    __syncwarp();
    const int piece = lane & 7;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int r = 4 * k + (lane >> 3);
      const int rt = __shfl_sync(0xffffffffu, tok, r);
      const float4 val = *reinterpret_cast<const float4*>(stage + r * kStageStride + 16 * piece);
      if (rt >= 0) red_add_v4(base + (int64_t)rt * 64 + 32 * h + 4 * piece, val.x, val.y, val.z, val.w);
    }
    __syncwarp();
  }
}

template <bool kCausal>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_tc_kernel(const __nv_bfloat16* __restrict__ qk, const __nv_bfloat16* __restrict__ v,
                   const __nv_bfloat16* __restrict__ dout, const int32_t* __restrict__ perm,
                   const float* __restrict__ lse, const float* __restrict__ Dg,
                   float* __restrict__ dqk, float* __restrict__ dv, int L, int n_rounds,
                   float scale, float scale_log2, int n_units, int units_per_seg,
                   int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* slots = smem;
  uint8_t* dsb = slots + kSlots * kSlotBytes;
  static_assert(8 * 32 * kStageStride <= 3 * kDsBlock, "flush staging fits in the dS^T blocks");
  BwdBar* bar = (BwdBar*)(dsb + kDsBytes);
  volatile int* abort = &bar->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_chunks = L / kM;
  const int n_pairs = (n_chunks + 1) / 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&bar->slot_full[s], 128);
      mbar_init(&bar->slot_free[s], 1);
    }
    mbar_init(&bar->s_full, 1);
    mbar_init(&bar->p_full, 256);
    mbar_init(&bar->g_full, 1);
    mbar_init(&bar->g_free, 256);
    mbar_init(&bar->mma_done, 1);
    bar->abort = 0;
    fence_mbar_init();
  }
  // the zero block after dS^T block 2 (rows of the R1 operand that must add 0)
  for (int i = threadIdx.x; i < kDsBlock / 16; i += kThreads)
    reinterpret_cast<uint4*>(dsb + 3 * kDsBlock)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async();
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
    const int t = threadIdx.x, row = t >> 1, half = t & 1;
    JobIter it(blockIdx.x, n_units, gridDim.x, units_per_seg, n_pairs);
    Job j;
    int n = 0;
    while (it.next(j)) {
      const int s = n % kSlots;
      if (n >= kSlots &&
          !mbar_wait(&bar->slot_free[s], (uint32_t)(n / kSlots - 1) & 1u, abort, status))
        break;
      const int64_t bh = j.seg / n_rounds;
      const int nc = min(3, n_chunks - 2 * j.p);     // chunks 2p .. 2p+nc-1 exist
      uint8_t* sl = slots + s * kSlotBytes;
      const __nv_bfloat16* xb = qk + bh * L * 64;
      const __nv_bfloat16* vb = v + bh * L * 64;
      const __nv_bfloat16* gb = dout + bh * L * 64;
      int pos[3];
      float l2[3], dd[3];
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        pos[c] = 0;
        if (c < nc) {
          int ps = perm[j.seg * L + (int64_t)(2 * j.p + c) * kM + row];
          if ((unsigned)ps >= (unsigned)L) {
            if (status) atomicExch(status, (int)LSH_ERR_DEVICE_CHECK);
            ps = 0;
          }
          pos[c] = ps;
        }
      }
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        if (c < nc) {
          issue_row(xb + (int64_t)pos[c] * 64, sl + kX + c * kTile, row, half);
          issue_row(gb + (int64_t)pos[c] * 64, sl + kDo + c * kTile, row, half);
          if (c < 2) issue_row(vb + (int64_t)pos[c] * 64, sl + kV + c * kTile, row, half);
        }
      }
      cp_async_commit();
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        l2[c] = 0.f;
        dd[c] = 0.f;
        if (c < nc && half == 0) {
          const float lv = lse[bh * L + pos[c]];
          l2[c] = (lv == -INFINITY) ? INFINITY : lv * kLog2e;
          dd[c] = Dg[bh * L + pos[c]];
        }
      }
      cp_async_wait<0>();
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        if (c < nc) {
          convert_row(sl + kX + c * kTile, row, half);
          convert_row(sl + kDo + c * kTile, row, half);
          if (c < 2) convert_row(sl + kV + c * kTile, row, half);
          if (half == 0) {
            bar->qpos[s][c * 64 + row] = pos[c];
            bar->lse2[s][c * 64 + row] = l2[c];
            bar->dval[s][c * 64 + row] = dd[c];
          }
        }
      }
      fence_proxy_async();
      mbar_arrive(&bar->slot_full[s]);
      ++n;
    }
  } else if (warp == 4) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_kk = idesc_f16(128, 64, 0, false, false);   // both K-major
      const uint32_t idesc_kn = idesc_f16(128, 64, 0, false, true);    // B MN-major
      const uint32_t idesc_nn = idesc_f16(128, 64, 0, true, true);     // A and B MN-major
      const uint32_t slots_a = smem_u32(slots), ds_a = smem_u32(dsb);
      JobIter it(blockIdx.x, n_units, gridDim.x, units_per_seg, n_pairs);
      Job j;
      int n = 0;
      while (it.next(j)) {
        const int s = n % kSlots;
        if (!mbar_wait(&bar->slot_full[s], (uint32_t)(n / kSlots) & 1u, abort, status)) break;
        if (n >= 1 && !mbar_wait(&bar->g_free, (uint32_t)(n - 1) & 1u, abort, status)) break;
        tc_fence_after();
        const int nc = min(3, n_chunks - 2 * j.p);
        const uint32_t sl = slots_a + s * kSlotBytes;
        // S^T = X_K X_Q^T and dP^T = V_K dO_Q^T, one N=64 block per query chunk
#pragma unroll
        for (int qb = 0; qb < 3; ++qb) {
          if (qb >= nc) continue;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            mma_ss(tmem + kColS + qb * 64, smem_desc(sl + kX + ks * 32, 16, 1024),
                   smem_desc(sl + kX + qb * kTile + ks * 32, 16, 1024), idesc_kk, ks > 0);
            mma_ss(tmem + kColDp + qb * 64, smem_desc(sl + kV + ks * 32, 16, 1024),
                   smem_desc(sl + kDo + qb * kTile + ks * 32, 16, 1024), idesc_kk, ks > 0);
          }
        }
        mma_commit(&bar->s_full);
        if (!mbar_wait(&bar->p_full, (uint32_t)n & 1u, abort, status)) break;
        tc_fence_after();
        bool acc_v = false, acc_k = false;
#pragma unroll
        for (int qb = 0; qb < 3; ++qb) {
          if (qb >= nc) continue;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            // dV += P^T (TMEM) . dO_Q ; dK += dS^T (smem, K-major) . X_Q
            mma_ts(tmem + kColDv, tmem + kColP + qb * 32 + ks * 8,
                   smem_desc(sl + kDo + qb * kTile + ks * 2048, 8192, 1024), idesc_kn, acc_v);
            acc_v = true;
            mma_ss(tmem + kColDk, smem_desc(ds_a + qb * kDsBlock + ks * 32, 16, 1024),
                   smem_desc(sl + kX + qb * kTile + ks * 2048, 8192, 1024), idesc_kn, acc_k);
            acc_k = true;
          }
        }
        // query-side terms through the transposed reading of dS^T
        const int kkeys = nc >= 2 ? 8 : 4;       // K = keys present (16 per step)
        for (int ks = 0; ks < kkeys; ++ks) {
          mma_ss(tmem + kColR0, smem_desc(ds_a + ks * 2048, kDsBlock, 1024),
                 smem_desc(sl + kX + ks * 2048, 8192, 1024), idesc_nn, ks > 0);
          if (nc == 3)
            mma_ss(tmem + kColR1, smem_desc(ds_a + 2 * kDsBlock + ks * 2048, kDsBlock, 1024),
                   smem_desc(sl + kX + ks * 2048, 8192, 1024), idesc_nn, ks > 0);
        }
        mma_commit(&bar->g_full);
        mma_commit(&bar->slot_free[s]);
        ++n;
      }
      mma_commit(&bar->mma_done);
      int dummy = 0;
      mbar_wait(&bar->mma_done, 0, (volatile int*)&dummy, status);
    }
  } else {
    // ------------------------------------------------ key rows: P, dS, gradients
    const int kwg = (warp - 5) >> 2;           // 0: first query block, 1: second
    const int q = warp & 3;
    const int row = q * 32 + lane;             // key row = TMEM lane
    const bool odd_row = row >= 64;
    const int qb0 = odd_row ? 1 : 0;           // first query block of this key row
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t tl = tmem + lane_off;
    JobIter it(blockIdx.x, n_units, gridDim.x, units_per_seg, n_pairs);
    Job j;
    int n = 0;
    while (it.next(j)) {
      const int s = n % kSlots;
      if (!mbar_wait(&bar->s_full, (uint32_t)n & 1u, abort, status)) break;
      tc_fence_after();
      const int nc = min(3, n_chunks - 2 * j.p);
      const bool row_live = row < 64 * min(nc, 2);
      const int kpos = bar->qpos[s][row];
      // position of this lane's row of chunk 2p+2 (read now: the slot may be
      // refilled once the gradient MMAs are done)
      const int qpos2 = (nc == 3 && !odd_row) ? bar->qpos[s][128 + row] : 0;
      const int* qp_all = bar->qpos[s];
      const float* l2_all = bar->lse2[s];
      const float* d_all = bar->dval[s];
      {
        const int qb = qb0 + kwg;
        const bool blk_ok = qb < nc && row_live;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int col0 = qb * 64 + h * 32;
          uint32_t sv[32], pv[32];
          tmem_ld32(tl + kColS + col0, sv);
          tmem_ld32(tl + kColDp + col0, pv);
          tmem_ld_wait();
          uint32_t pk[16], dk[16];
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4) {
            int4 q4 = make_int4(0, 0, 0, 0);
            float4 l4 = make_float4(0.f, 0.f, 0.f, 0.f), d4 = l4;
            if (blk_ok) {
              q4 = *reinterpret_cast<const int4*>(qp_all + col0 + 4 * i4);
              l4 = *reinterpret_cast<const float4*>(l2_all + col0 + 4 * i4);
              d4 = *reinterpret_cast<const float4*>(d_all + col0 + 4 * i4);
            }
            const int qq[4] = {q4.x, q4.y, q4.z, q4.w};
            const float ll[4] = {l4.x, l4.y, l4.z, l4.w};
            const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
            float pe[4], de[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = 4 * i4 + e;
              const bool valid = blk_ok && (kCausal ? (kpos < qq[e]) : (kpos != qq[e]));
              const float pr = ex2(fmaf(__uint_as_float(sv[i]), scale_log2, -ll[e]));
              pe[e] = valid ? pr : 0.f;
              de[e] = valid ? pr * (__uint_as_float(pv[i]) - dd[e]) : 0.f;
            }
            pk[2 * i4] = pack_f16x2(pe[0], pe[1]);
            pk[2 * i4 + 1] = pack_f16x2(pe[2], pe[3]);
            dk[2 * i4] = pack_f16x2(de[0], de[1]);
            dk[2 * i4 + 1] = pack_f16x2(de[2], de[3]);
          }
          // P^T into TMEM (block qb at columns kColP + 32 qb), dS^T into smem
          tmem_st16(tl + kColP + (uint32_t)(qb * 32 + h * 16), pk);
          uint8_t* drow = dsb + qb * kDsBlock + row * 128;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int ch = h * 4 + c;
            *reinterpret_cast<uint4*>(drow + ((ch ^ (row & 7)) << 4)) =
                make_uint4(dk[4 * c], dk[4 * c + 1], dk[4 * c + 2], dk[4 * c + 3]);
          }
        }
      }
      if (kwg == 1) {
        // the query block this key row does not see: P = 0 and dS = 0
        const int zb = odd_row ? 0 : 2;
        uint32_t z[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) z[e] = 0u;
        tmem_st32(tl + kColP + (uint32_t)(zb * 32), z);
        uint8_t* drow = dsb + zb * kDsBlock + row * 128;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          *reinterpret_cast<uint4*>(drow + ((ch ^ (row & 7)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
      }
      tmem_st_wait();
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(&bar->p_full);
      // gradients of this pair
      if (!mbar_wait(&bar->g_full, (uint32_t)n & 1u, abort, status)) break;
      tc_fence_after();
      const int64_t bh = j.seg / n_rounds;
      // staging: the dS^T blocks are idle until the next item's softmax,
      // which starts only after every row here has been flushed
      uint8_t* stage = dsb + (warp - 5) * (32 * kStageStride);
      const int tok = row_live ? kpos : -1;
      if (kwg == 0) flush_rows(dv + bh * L * 64, tok, tl + kColDv, 0, false, 1.f, stage, lane);
      if (kwg == 1)
        flush_rows(dqk + bh * L * 64, tok, tl + kColDk, tl + kColR0, true, scale, stage, lane);
      if (kwg == 0 && nc == 3 && !odd_row) {
        // query-side term of chunk 2p+2 (lanes 0..63 of R1)
        flush_rows(dqk + bh * L * 64, qpos2, tl + kColR1, 0, false, scale, stage, lane);
      }
      tc_fence_before();
      mbar_arrive(&bar->g_free);
      ++n;
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

cudaError_t launch_attn_bwd_tc(const lsh_problem& p, const void* qk, const void* v,
                               const void* dout, const int32_t* perm, const float* lse,
                               const float* D, float* dqk, float* dv, int* status, cudaStream_t s) {
  if (p.dtype != LSH_BF16 || p.chunk != kM || !(p.scale > 0.f)) return cudaErrorNotSupported;
  const int n_chunks = p.L / kM;
  const int n_pairs = (n_chunks + 1) / 2;
  const int units_per_seg = (n_pairs + kUnit - 1) / kUnit;
  const int64_t n_units = (int64_t)p.B * p.H * p.n_rounds * units_per_seg;
  if (n_units > INT32_MAX) return cudaErrorNotSupported;
  int grid = sm_count();
  if ((int64_t)grid > n_units) grid = (int)n_units;
  auto kern = p.causal ? attn_bwd_tc_kernel<true> : attn_bwd_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kSmemBytes, s>>>(
      (const __nv_bfloat16*)qk, (const __nv_bfloat16*)v, (const __nv_bfloat16*)dout, perm, lse, D,
      dqk, dv, p.L, p.n_rounds, p.scale, p.scale * kLog2e, (int)n_units, units_per_seg, status);
  note_launch();
  return cudaGetLastError();
}

}  // namespace lsh
