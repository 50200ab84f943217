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
// segment — 128 keys, one per TMEM lane. The queries that see them are
// chunks 2p, 2p+1, 2p+2 (chunk c sees chunks c-1 and c): three query blocks
// of 64; key rows of chunk 2p see blocks 0-1, rows of chunk 2p+1 blocks 1-2.
// Each block is one pipeline step, in the order 1, 0, 2 (the block that all
// 128 key rows see, whose softmax is the longest, goes first):
//   S^T = X_K X_qb^T, dP^T = V_K dO_qb^T        (M=128 keys, N=64)
//   P^T and dS^T (fp16, in place over S^T and dP^T in TMEM; dS^T also to
//   shared memory for the query-side products)
//   dV += P^T dO_qb,  dK += dS^T X_qb           (A from TMEM, accumulated in TMEM)
// and once blocks 1 and 0 / block 2 are done, the query-side terms through the
// transposed (MN-major) reading of the dS^T tiles:
//   R0 = dS[blocks 0,1] X_K — for chunks 2p, 2p+1, i.e. the same tokens as
//        the key rows, lane for lane: accumulated straight into dK;
//   R1 = dS[block 2, zeros] X_K — for chunk 2p+2, which is the first key
//        chunk of the next pair: written into the OTHER accumulator set's dK,
//        so that the next item of the same unit adds its own terms on top.
//        At the end of a unit it is stored on its own (the edge rows below).
// The finished rows dV and scale*dK of an item are stored, converted to fp16,
// as per-round partial gradients in token order: each key row's two 128-byte
// rows go to the row's position, so every round's partial is a plain
// (position, 64) array. Unit-end R1 rows go to a small
// edge buffer, and the first item of the next unit records, per position of
// its first chunk, which edge row belongs to it (-1 for every other
// position). A second kernel then streams the rounds' partials of every
// token, adds its edge rows and writes dqk and dv, so no atomics and no
// inverse permutation are needed.
//
// TMEM (512 columns): two S^T|dP^T buffers (steps alternate) and two
// dV|dK accumulator sets (items alternate), so that the S^T/dP^T products
// of the next step, the softmax of this one and the flush of the previous
// item all run at once.
//
// Warp roles (persistent CTA, one per SM), register budgets via setmaxnreg:
//   warps 0-2  : producers — cp.async gathers of the fp16 copies of x, dout
//                (3 chunks) and v (2 chunks) into a 2-slot ring, per-query
//                position, log2-scaled LSE and D;
//   warp 3     : TMEM allocation and the MMA issue (the warp waits
//                converged; one elected lane issues each MMA and commit);
//   warps 4-7  : gradient flush of the previous item (one thread per key
//                row: TMEM -> fp16 -> a padded staging row; then each warp
//                stores its 32 rows, four whole rows per store instruction,
//                at their places in the partial arrays);
//   warps 8-23 : four softmax warpgroups, two per S^T buffer (even and odd
//                steps), one thread per key row and 32 of the block's 64
//                query columns each.
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
constexpr int kStageRow = 144;         // fp16 row of 128 bytes + 16 bytes of padding
constexpr int kStageBytes = 128 * kStageRow;
constexpr int kThreads = 768;
constexpr int kProducers = 96;
// Launched at 80 registers per thread (768 threads); producers/MMA and flush
// drop to 48, the four softmax warpgroups rise to 96.
constexpr int kRegsLaunch = 80;
constexpr int kRegsLow = 48, kRegsFlush = 48, kRegsSmx = 96;
static_assert(128 * (kRegsLow + kRegsFlush) + 512 * kRegsSmx <= kThreads * kRegsLaunch,
              "register split");
// TMEM columns
constexpr uint32_t kColBuf = 0;        // + 128 w: S^T (64) | dP^T (64); P^T over S^T
constexpr uint32_t kColAcc = 256;      // + 128 a: dV (64) | dK (64)

struct __align__(16) BwdBar {
  uint64_t slot_full[kSlots];
  uint64_t slot_free[kSlots];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t g_full[2];
  uint64_t acc_free[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  alignas(16) int qpos[kSlots][192];     // positions of query columns (= key rows for 0..127)
  alignas(16) float lse2[kSlots][192];   // LSE * log2(e); +inf for self-attending rows
  alignas(16) float dval[kSlots][192];   // D = dout . out
  alignas(16) int tok[4][192];           // positions again, per item (read by the flush)
};
static_assert(offsetof(BwdBar, qpos) % 16 == 0 && offsetof(BwdBar, lse2) % 16 == 0 &&
                  offsetof(BwdBar, dval) % 16 == 0,
              "per-column arrays are read with 16-byte loads");

constexpr size_t kSmemBytes =
    1024 + kSlots * kSlotBytes + kDsBytes + kStageBytes + sizeof(BwdBar);
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

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
// A wait's outcome made uniform across the warp, so that a timeout seen by
// one lane never leaves the others inside a warp-collective instruction.
__device__ __forceinline__ bool warp_ok(bool ok) { return __all_sync(0xffffffffu, ok); }

// Converts 64 fp32 TMEM columns of this thread's lane, times `sc`, to fp16
// into the thread's row of its warp's 32 staging rows (144 bytes apart, so the
// 16-byte stores of eight consecutive rows fall in different banks); then the
// warp copies the 32 rows out, four whole 128-byte rows per store instruction
// (eight lanes of 16 bytes each): row k goes to base + lane k's `off`
// (halves), unless lane k's `live` is false.
__device__ __forceinline__ void put_rows(uint32_t ta, float sc, uint8_t* wstage, int lane,
                                         __half* base, int64_t off, bool live) {
  uint8_t* srow = wstage + lane * kStageRow;
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    uint32_t a[16];
    tmem_ld16(ta + 16 * h, a);
    tmem_ld_wait();
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      pk[i] = pack_f16x2(__uint_as_float(a[2 * i]) * sc, __uint_as_float(a[2 * i + 1]) * sc);
    uint4* d = reinterpret_cast<uint4*>(srow) + 2 * h;
    d[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    d[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  }
  __syncwarp();
  const int sub = lane >> 3, ch = lane & 7;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int k = 4 * i + sub;
    const long long ok = __shfl_sync(0xffffffffu, (long long)off, k);
    const int lk = __shfl_sync(0xffffffffu, live ? 1 : 0, k);
    if (lk) {
      const uint4 v = *reinterpret_cast<const uint4*>(wstage + k * kStageRow + ch * 16);
      *reinterpret_cast<uint4*>(base + ok + ch * 8) = v;
    }
  }
  __syncwarp();
}

// ---- MMA issue helpers (one thread). Descriptor lower words: `sl` is the
// slot's shared address >> 4; LBO fields are added per operand layout.
constexpr uint32_t kIdKK = idesc_f16(128, 64, 0, false, false);   // A, B K-major
constexpr uint32_t kIdKN = idesc_f16(128, 64, 0, false, true);    // B MN-major
constexpr uint32_t kIdNN = idesc_f16(128, 64, 0, true, true);     // A, B MN-major
constexpr uint32_t kLboK = desc_lbo(16), kLboN = desc_lbo(kTile);

// S^T = X_K X_qb^T and dP^T = V_K dO_qb^T of step g (buffer g & 1); commits `full`.
__device__ __forceinline__ void bwd_issue_s(uint32_t tmem, uint32_t sl, int g, int qb, int nc,
                                            uint64_t* full) {
  if (elect_one()) {
    if (qb < nc) {
      const uint32_t d = tmem + kColBuf + (uint32_t)(g & 1) * 128;
      const uint32_t xk = sl + kX / 16 + kLboK, vk = sl + kV / 16 + kLboK;
      const uint32_t xq = sl + (kX + qb * kTile) / 16 + kLboK, gq = sl + (kDo + qb * kTile) / 16 + kLboK;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        mma_ss_raw(d, xk + 2 * ks, xq + 2 * ks, kDescHi1024, kIdKK, ks > 0);
        mma_ss_raw(d + 64, vk + 2 * ks, gq + 2 * ks, kDescHi1024, kIdKK, ks > 0);
      }
    }
    mma_commit_raw(full);
  }
  __syncwarp();
}
// dV += P^T dO_qb ; dK += dS^T X_qb, P^T and dS^T from step g's TMEM buffer.
__device__ __forceinline__ void bwd_issue_g(uint32_t tmem, uint32_t acc, uint32_t sl, int g, int qb,
                                            bool acc_v, bool acc_k) {
  const uint32_t pt = tmem + kColBuf + (uint32_t)(g & 1) * 128;
  const uint32_t gq = sl + (kDo + qb * kTile) / 16 + kLboN, xq = sl + (kX + qb * kTile) / 16 + kLboN;
  // packed queries 0-31 sit at columns 0-15, queries 32-63 at columns 32-47
  if (elect_one()) {
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const uint32_t ca = 8 * ks + 16 * (ks >> 1);
      mma_ts_raw(acc, pt + ca, gq + 128 * ks, kDescHi1024, kIdKN, acc_v || ks > 0);
      mma_ts_raw(acc + 64, pt + 64 + ca, xq + 128 * ks, kDescHi1024, kIdKN, acc_k || ks > 0);
    }
  }
  __syncwarp();
}
// Query-side product dS[128 queries of the dS^T blocks at ds] X_K over the
// keys [16 KS0, 16 KS1), into the dK columns at d.
template <int KS0, int KS1>
__device__ __forceinline__ void bwd_issue_r(uint32_t d, uint32_t ds, uint32_t sl, bool acc) {
  const uint32_t xk = sl + kX / 16 + kLboN;
  if (elect_one()) {
#pragma unroll
    for (int ks = KS0; ks < KS1; ++ks)
      mma_ss_raw(d, ds + 128 * ks, xk + 128 * ks, kDescHi1024, kIdNN, acc || ks > KS0);
  }
  __syncwarp();
}
__device__ __forceinline__ bool bwd_wait_p(BwdBar* bar, int g, volatile int* abort, int* status) {
  return __all_sync(0xffffffffu, mbar_wait(&bar->p_full[g & 1], (uint32_t)(g >> 1) & 1u, abort, status));
}

template <bool kCausal>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_tc_kernel(const __half* __restrict__ qk, const __half* __restrict__ v,
                   const __half* __restrict__ dout, const int32_t* __restrict__ perm,
                   const float* __restrict__ lse, const float* __restrict__ Dg,
                   __half* __restrict__ part_dv, __half* __restrict__ part_dqk,
                   __half* __restrict__ edge, int32_t* __restrict__ emap, int L, int n_rounds,
                   float scale, float scale_log2, int n_units, int units_per_seg,
                   int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* slots = smem;
  uint8_t* dsb = slots + kSlots * kSlotBytes;
  uint8_t* stage = dsb + kDsBytes;
  BwdBar* bar = (BwdBar*)(stage + kStageBytes);
  volatile int* abort = &bar->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_chunks = L / kM;
  const int n_pairs = (n_chunks + 1) / 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&bar->slot_full[s], kProducers);
      mbar_init(&bar->slot_free[s], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&bar->s_full[w], 1);
      mbar_init(&bar->p_full[w], 256);
      mbar_init(&bar->g_full[w], 1);
      mbar_init(&bar->acc_free[w], 128);
    }
    mbar_init(&bar->mma_done, 1);
    bar->abort = 0;
    fence_mbar_init();
  }
  // the zero block after dS^T block 2 (rows of the R1 operand that must add 0)
  for (int i = threadIdx.x; i < kDsBlock / 16; i += kThreads)
    reinterpret_cast<uint4*>(dsb + 3 * kDsBlock)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async();
  if (warp == 3) {
    tmem_alloc(&bar->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  const int wgi = warp >> 2;

  if (wgi == 0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
    if (warp < 3) {
      // ---------------------------------------------- producers: warp c gathers
      // chunk 2p+c (x, dout, and v for c < 2). Eight lanes cover one 128-byte
      // row, so each cp.async instruction moves four whole rows.
      const int c = warp;
      const int ch = lane & 7, rsub = lane >> 3;
      JobIter it(blockIdx.x, n_units, gridDim.x, units_per_seg, n_pairs);
      Job j, jn;
      bool have = it.next(j);
      // positions of rows lane and 32+lane of chunk 2p+c, loaded one item ahead
      auto load_pos = [&](const Job& jj, int& pa, int& pb) {
        pa = pb = 0;
        if (c < min(3, n_chunks - 2 * jj.p)) {
          const int32_t* pj = perm + jj.seg * L + (int64_t)(2 * jj.p + c) * kM;
          pa = __ldg(pj + lane);
          pb = __ldg(pj + 32 + lane);
        }
      };
      int pa = 0, pb = 0;
      if (have) load_pos(j, pa, pb);
      int n = 0;
      while (have) {
        const bool have_next = it.next(jn);
        int pa_n = 0, pb_n = 0;
        if (have_next) load_pos(jn, pa_n, pb_n);
        const int s = n % kSlots;
        if (n >= kSlots &&
            !warp_ok(mbar_wait(&bar->slot_free[s], (uint32_t)(n / kSlots - 1) & 1u, abort, status)))
          break;
        const int64_t bh = j.seg / n_rounds;
        const bool live = c < min(3, n_chunks - 2 * j.p);
        uint8_t* sl = slots + s * kSlotBytes;
        if ((unsigned)pa >= (unsigned)L || (unsigned)pb >= (unsigned)L) {
          record_status(status, (int)LSH_ERR_DEVICE_CHECK);
          if ((unsigned)pa >= (unsigned)L) pa = 0;
          if ((unsigned)pb >= (unsigned)L) pb = 0;
        }
        if (live) {
          const __half* xb = qk + bh * L * 64 + ch * 8;
          const __half* gb = dout + bh * L * 64 + ch * 8;
          const __half* vb = v + bh * L * 64 + ch * 8;
          const uint32_t tx = smem_u32(sl + kX + c * kTile), tg = smem_u32(sl + kDo + c * kTile),
                         tv = smem_u32(sl + kV + c * kTile);
#pragma unroll
          for (int g = 0; g < 16; ++g) {
            const int row = 4 * g + rsub;
            const int64_t pos = __shfl_sync(0xffffffffu, g < 8 ? pa : pb, row & 31);
            const uint32_t off = row * 128 + (((uint32_t)ch ^ (uint32_t)(row & 7)) << 4);
            cp_async16(tx + off, xb + pos * 64);
            cp_async16(tg + off, gb + pos * 64);
            if (c < 2) cp_async16(tv + off, vb + pos * 64);
          }
        }
        cp_async_commit();
        // per query column: position, LSE, D (while the rows are in flight)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int q = c * 64 + k * 32 + lane;
          const int pos = k ? pb : pa;
          int tp = -1;
          float l2 = 0.f, dd = 0.f;
          if (live) {
            const float lv = lse[bh * L + pos];
            l2 = (lv == -INFINITY) ? INFINITY : lv * kLog2e;
            dd = Dg[bh * L + pos];
            tp = pos;
          }
          bar->qpos[s][q] = tp;
          bar->lse2[s][q] = l2;
          bar->dval[s][q] = dd;
          bar->tok[n & 3][q] = tp;
        }
        cp_async_wait<0>();
        fence_proxy_async();
        mbar_arrive(&bar->slot_full[s]);
        j = jn;
        pa = pa_n;
        pb = pb_n;
        have = have_next;
        ++n;
      }
    } else {
      // ---------------------------------------------- MMA issuer (whole warp
      // converged; each MMA / commit issued by one elected lane)
      JobIter it(blockIdx.x, n_units, gridDim.x, units_per_seg, n_pairs);
      Job cur, nxt;
      bool have = it.next(cur);
      bool ok = true;
      const uint32_t slot0 = smem_u32(slots) >> 4;
      const uint32_t ds_lo = (smem_u32(dsb) >> 4) | desc_lbo(kDsBlock);
      int seen0 = 0, seen1 = 0;   // acc_free completions waited for, per set
      if (have) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bar->slot_full[0], 0u, abort, status));
        if (ok) {
          tc_fence_after();
          const int nc = min(3, n_chunks - 2 * cur.p);
          bwd_issue_s(tmem, slot0, 0, 1, nc, &bar->s_full[0]);
          bwd_issue_s(tmem, slot0, 1, 0, nc, &bar->s_full[1]);
        }
      }
      int n = 0;
      bool prev_r1_alone = false;   // the previous item left R1 rows for its own flush
      while (ok && have) {
        const bool have_next = it.next(nxt);
        const int s = n % kSlots, a = n & 1;
        const int nc = min(3, n_chunks - 2 * cur.p);
        const uint32_t sl = slot0 + (uint32_t)(s * kSlotBytes) / 16;
        const uint32_t acc = tmem + kColAcc + (uint32_t)a * 128;
        const int g0 = 3 * n;
        // ---- step 0: query block 1 (the one all 128 key rows see)
        if (!bwd_wait_p(bar, g0, abort, status)) break;
        // flushes of the earlier items that used set a (and, after a unit's
        // last item, of that item too: it read its R1 rows from set a)
        {
          const int need = n >> 1;
          int& seen = a ? seen1 : seen0;
          while (ok && seen < need)
            ok = __all_sync(0xffffffffu, mbar_wait(&bar->acc_free[a], (uint32_t)(seen++) & 1u, abort, status));
          if (prev_r1_alone) {
            const int b = a ^ 1, need_b = ((n - 1) >> 1) + 1;
            int& seen_b = b ? seen1 : seen0;
            while (ok && seen_b < need_b)
              ok = __all_sync(0xffffffffu, mbar_wait(&bar->acc_free[b], (uint32_t)(seen_b++) & 1u, abort, status));
          }
          if (!ok) break;
        }
        tc_fence_after();
        if (nc > 1) bwd_issue_g(tmem, acc, sl, g0, 1, false, !cur.first);
        bwd_issue_s(tmem, sl, g0 + 2, 2, nc, &bar->s_full[(g0 + 2) & 1]);
        // ---- step 1: query block 0, then R0 = dS[blocks 0,1] X_K into dK
        if (!bwd_wait_p(bar, g0 + 1, abort, status)) break;
        tc_fence_after();
        bwd_issue_g(tmem, acc, sl, g0 + 1, 0, nc > 1, nc > 1 || !cur.first);
        if (nc >= 2) bwd_issue_r<0, 8>(acc + 64, ds_lo, sl, true);
        else bwd_issue_r<0, 4>(acc + 64, ds_lo, sl, true);
        int nc_next = 0;
        uint32_t sl_next = 0;
        if (have_next) {
          const int sn = (n + 1) % kSlots;
          if (!__all_sync(0xffffffffu, mbar_wait(&bar->slot_full[sn], (uint32_t)((n + 1) / kSlots) & 1u, abort, status)))
            break;
          tc_fence_after();
          nc_next = min(3, n_chunks - 2 * nxt.p);
          sl_next = slot0 + (uint32_t)(sn * kSlotBytes) / 16;
          bwd_issue_s(tmem, sl_next, g0 + 3, 1, nc_next, &bar->s_full[(g0 + 3) & 1]);
        }
        // ---- step 2: query block 2, then R1 = dS[block 2, zeros] X_K into the other set's dK
        if (!bwd_wait_p(bar, g0 + 2, abort, status)) break;
        tc_fence_after();
        if (nc == 3) {
          bwd_issue_g(tmem, acc, sl, g0 + 2, 2, true, true);
          const int b = a ^ 1, need_b = (n + 1) >> 1;
          int& seen_b = b ? seen1 : seen0;
          while (ok && seen_b < need_b)
            ok = __all_sync(0xffffffffu, mbar_wait(&bar->acc_free[b], (uint32_t)(seen_b++) & 1u, abort, status));
          if (!ok) break;
          tc_fence_after();
          // block 2's queries see only the keys of chunk 2p+1 (rows 64-127;
          // the other rows of the block hold zeros)
          bwd_issue_r<4, 8>(tmem + kColAcc + (uint32_t)b * 128 + 64, ds_lo + 2 * (kDsBlock / 16), sl,
                            false);
        }
        mma_commit(&bar->g_full[a]);
        mma_commit(&bar->slot_free[s]);
        prev_r1_alone = cur.last && nc == 3;
        if (have_next)
          bwd_issue_s(tmem, sl_next, g0 + 4, 0, nc_next, &bar->s_full[(g0 + 4) & 1]);
        cur = nxt;
        have = have_next;
        ++n;
      }
      mma_commit(&bar->mma_done);
      int dummy = 0;
      mbar_wait(&bar->mma_done, 0, (volatile int*)&dummy, status);
    }
  } else if (wgi == 1) {
    // ------------------------------------------------ gradient flush
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsFlush));
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
    uint8_t* wstage = stage + q * 32 * kStageRow;
    JobIter it(blockIdx.x, n_units, gridDim.x, units_per_seg, n_pairs);
    Job j;
    int n = 0;
    while (it.next(j)) {
      const int a = n & 1;
      if (!warp_ok(mbar_wait(&bar->g_full[a], (uint32_t)(n >> 1) & 1u, abort, status))) break;
      tc_fence_after();
      const int nc = min(3, n_chunks - 2 * j.p);
      const bool live = row < 64 * min(nc, 2);   // key rows present
      const int tp = bar->tok[n & 3][row];        // this key row's position
      const int64_t rr = j.seg * L + (live ? tp : 0);
      const uint32_t acc = tl + kColAcc + (uint32_t)a * 128;
      const bool r1 = j.last && nc == 3;
      const int unit = (int)(j.seg * units_per_seg + j.p / kUnit);
      put_rows(acc, 1.f, wstage, lane, part_dv, rr * 64, live);
      put_rows(acc + 64, scale, wstage, lane, part_dqk, rr * 64, live);
      // the rows of a unit's first chunk (after the first unit) take the R1
      // rows that the previous unit's last item stored on its own
      if (live) emap[rr] = (j.first && j.p > 0 && row < kM) ? (unit - 1) * kM + row : -1;
      if (r1 && q < 2)
        put_rows(tl + kColAcc + (uint32_t)(a ^ 1) * 128 + 64, scale, wstage, lane, edge,
                 ((int64_t)unit * kM + row) * 64, true);
      tc_fence_before();
      mbar_arrive(&bar->acc_free[a]);
      ++n;
    }
  } else {
    // ------------------------------------------------ softmax: P^T and dS^T
    // Two warpgroups per S^T buffer, each owning 32 of the block's 64 query
    // columns; each writes its packed P^T / dS^T inside its own half of the
    // buffer's columns, so neither overwrites columns the other still reads.
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSmx));
    const int sw = wgi - 2;
    const int w = sw >> 1;                     // S^T buffer = parity of the step
    const int hc = sw & 1;                     // column half of the block
    const int q = warp & 3;
    const int row = q * 32 + lane;             // key row = TMEM lane
    const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + kColBuf + (uint32_t)w * 128 +
                        (uint32_t)(32 * hc);
    JobIter it(blockIdx.x, n_units, gridDim.x, units_per_seg, n_pairs);
    Job j;
    int n = 0, k = 0;
    bool ok = true;
    while (ok && it.next(j)) {
      const int s = n % kSlots;
      const int nc = min(3, n_chunks - 2 * j.p);
      for (int kstep = 0; kstep < 3; ++kstep) {
        // steps of an item take query blocks 1, 0, 2 (the full block first)
        const int qb = kstep == 0 ? 1 : (kstep == 1 ? 0 : 2);
        if (((3 * n + kstep) & 1) != w) continue;
        if (!warp_ok(mbar_wait(&bar->s_full[w], (uint32_t)k & 1u, abort, status))) {
          ok = false;
          break;
        }
        ++k;
        tc_fence_after();
        if (qb < nc) {
          const bool active = qb == 1 || (qb == 0 ? row < 64 : row >= 64);
          uint8_t* drow = dsb + qb * kDsBlock + row * 128;
          if (active) {
            const int kpos = bar->qpos[s][row];  // this key row's position
            const int* qp_all = bar->qpos[s];
            const float* l2_all = bar->lse2[s];
            const float* d_all = bar->dval[s];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int col0 = qb * 64 + 32 * hc + 16 * h;
              uint32_t sv[16], pv[16];
              tmem_ld16(tb + 16 * h, sv);
              tmem_ld16(tb + 64 + 16 * h, pv);
              tmem_ld_wait();
              uint32_t pk[8], dk[8];
#pragma unroll
              for (int i4 = 0; i4 < 4; ++i4) {
                const int4 q4 = *reinterpret_cast<const int4*>(qp_all + col0 + 4 * i4);
                const float4 l4 = *reinterpret_cast<const float4*>(l2_all + col0 + 4 * i4);
                const float4 d4 = *reinterpret_cast<const float4*>(d_all + col0 + 4 * i4);
                const int qq[4] = {q4.x, q4.y, q4.z, q4.w};
                const float ll[4] = {l4.x, l4.y, l4.z, l4.w};
                const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
                float pe[4], de[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int i = 4 * i4 + e;
                  const bool valid = kCausal ? (kpos < qq[e]) : (kpos != qq[e]);
                  const float pr = ex2(fmaf(__uint_as_float(sv[i]), scale_log2, -ll[e]));
                  pe[e] = valid ? pr : 0.f;
                  // pe is 0 where masked and dP - D is finite, so no second select
                  de[e] = pe[e] * (__uint_as_float(pv[i]) - dd[e]);
                }
                pk[2 * i4] = pack_f16x2(pe[0], pe[1]);
                pk[2 * i4 + 1] = pack_f16x2(pe[2], pe[3]);
                dk[2 * i4] = pack_f16x2(de[0], de[1]);
                dk[2 * i4 + 1] = pack_f16x2(de[2], de[3]);
              }
              // packed P^T and dS^T over this half's S^T / dP^T columns that
              // are already read; dS^T also into shared memory
              tmem_st8(tb + 8 * h, pk);
              tmem_st8(tb + 64 + 8 * h, dk);
#pragma unroll
              for (int c = 0; c < 2; ++c) {
                const int ch = 4 * hc + 2 * h + c;
                *reinterpret_cast<uint4*>(drow + ((ch ^ (row & 7)) << 4)) =
                    make_uint4(dk[4 * c], dk[4 * c + 1], dk[4 * c + 2], dk[4 * c + 3]);
              }
            }
          } else {
            // a key row that this query block does not see: P = 0 and dS = 0
            uint32_t z[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) z[e] = 0u;
            tmem_st16(tb, z);
            tmem_st16(tb + 64, z);
#pragma unroll
            for (int c = 0; c < 4; ++c)
              *reinterpret_cast<uint4*>(drow + (((4 * hc + c) ^ (row & 7)) << 4)) =
                  make_uint4(0u, 0u, 0u, 0u);
          }
          tmem_st_wait();
          fence_proxy_async();
        }
        tc_fence_before();
        mbar_arrive(&bar->p_full[w]);
      }
      ++n;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 3) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// D_i = dout_i . (out_i + out_lo_i), and fp16 copies of qk, v and dout for the
// tensor-core products (exact for values inside the fp16 range; a value
// outside it becomes inf, which the check of the results reports). Eight
// threads per token, 16 bytes of each tensor per thread.
__global__ void __launch_bounds__(256)
bwd_prep_tc_kernel(const __nv_bfloat16* __restrict__ qk, const __nv_bfloat16* __restrict__ v,
                   const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ out,
                   const __nv_bfloat16* __restrict__ out_lo, float* __restrict__ D,
                   __half* __restrict__ x16, __half* __restrict__ v16, __half* __restrict__ g16,
                   int64_t N) {
  const int64_t tok = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 3;
  const int c8 = (threadIdx.x & 7) * 8;
  const bool live = tok < N;
  const int64_t off = (live ? tok : 0) * 64 + c8;
  uint4 o = make_uint4(0u, 0u, 0u, 0u), lo = o, g = o, x = o, w = o;
  if (live) {
    o = __ldg(reinterpret_cast<const uint4*>(out + off));
    if (out_lo) lo = __ldg(reinterpret_cast<const uint4*>(out_lo + off));
    g = __ldg(reinterpret_cast<const uint4*>(dout + off));
    x = __ldg(reinterpret_cast<const uint4*>(qk + off));
    w = __ldg(reinterpret_cast<const uint4*>(v + off));
  }
  const uint32_t ou[4] = {o.x, o.y, o.z, o.w}, lu[4] = {lo.x, lo.y, lo.z, lo.w};
  const uint32_t gu[4] = {g.x, g.y, g.z, g.w};
  float d = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float o0 = __uint_as_float(ou[i] << 16) + __uint_as_float(lu[i] << 16);
    const float o1 = __uint_as_float(ou[i] & 0xffff0000u) + __uint_as_float(lu[i] & 0xffff0000u);
    d = fmaf(o0, __uint_as_float(gu[i] << 16), d);
    d = fmaf(o1, __uint_as_float(gu[i] & 0xffff0000u), d);
  }
  d += __shfl_xor_sync(0xffffffffu, d, 4);
  d += __shfl_xor_sync(0xffffffffu, d, 2);
  d += __shfl_xor_sync(0xffffffffu, d, 1);
  if (!live) return;
  if (c8 == 0) D[tok] = d;
  *reinterpret_cast<uint4*>(x16 + off) = make_uint4(bf16x2_to_f16x2(x.x), bf16x2_to_f16x2(x.y),
                                                    bf16x2_to_f16x2(x.z), bf16x2_to_f16x2(x.w));
  *reinterpret_cast<uint4*>(v16 + off) = make_uint4(bf16x2_to_f16x2(w.x), bf16x2_to_f16x2(w.y),
                                                    bf16x2_to_f16x2(w.z), bf16x2_to_f16x2(w.w));
  *reinterpret_cast<uint4*>(g16 + off) = make_uint4(bf16x2_to_f16x2(g.x), bf16x2_to_f16x2(g.y),
                                                    bf16x2_to_f16x2(g.z), bf16x2_to_f16x2(g.w));
}

__device__ __forceinline__ void add8_f16(float (&acc)[8], const uint4 w) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[i]));
    acc[2 * i] += f.x;
    acc[2 * i + 1] += f.y;
  }
}

// Eight floats to a 32-byte aligned address in one store.
__device__ __forceinline__ void st_global_v8f(float* p, const float (&w)[8]) {
  asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "f"(w[0]),
               "f"(w[1]), "f"(w[2]), "f"(w[3]), "f"(w[4]), "f"(w[5]), "f"(w[6]), "f"(w[7])
               : "memory");
}

// dv, dqk of every token: the sum over rounds of its partial rows (row pos
// of segment bh * n_rounds + r), plus the R1 row that emap names where the
// token opens a unit; dv also takes dout for a token that attended only to
// itself (final LSE of -inf). Eight threads per token; the rows of two
// rounds are loaded together, to keep more reads in flight.
__global__ void __launch_bounds__(256)
sum_rounds_kernel(const __half* __restrict__ part_dv, const __half* __restrict__ part_dqk,
                  const __half* __restrict__ edge, const int32_t* __restrict__ emap,
                  const float* __restrict__ lse, const __nv_bfloat16* __restrict__ dout,
                  float* __restrict__ dqk, float* __restrict__ dv, int L, int n_rounds,
                  int64_t n_edge_rows, int64_t N, int wide, int* status) {
  const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 3;
  const int c8 = (threadIdx.x & 7) * 8;
  if (t >= N) return;
  const int64_t bh = t / L;
  const int pos = (int)(t - bh * L);
  float a[8], b[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) a[e] = b[e] = 0.f;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  for (int r0 = 0; r0 < n_rounds; r0 += 2) {
    uint4 ua[2], ub[2];
    int er[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const bool live = r0 + k < n_rounds;
      const int64_t row = (bh * n_rounds + (live ? r0 + k : 0)) * L + pos;
      ua[k] = live ? __ldg(reinterpret_cast<const uint4*>(part_dv + row * 64 + c8)) : zero;
      ub[k] = live ? __ldg(reinterpret_cast<const uint4*>(part_dqk + row * 64 + c8)) : zero;
      er[k] = live ? __ldg(emap + row) : -1;
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      add8_f16(a, ua[k]);
      add8_f16(b, ub[k]);
      if (er[k] >= 0) {
        if (er[k] < n_edge_rows)
          add8_f16(b, __ldg(reinterpret_cast<const uint4*>(edge + (int64_t)er[k] * 64 + c8)));
        else
          record_status(status, (int)LSH_ERR_DEVICE_CHECK);
      }
    }
  }
  if (lse[t] == -INFINITY) {
    const uint4 w = *reinterpret_cast<const uint4*>(dout + t * 64 + c8);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      a[2 * i] += __uint_as_float(u[i] << 16);
      a[2 * i + 1] += __uint_as_float(u[i] & 0xffff0000u);
    }
  }
  // the partial rows are fp16: a value outside its range (or a non-finite
  // input) leaves a non-finite gradient, which is reported
  bool fin = true;
#pragma unroll
  for (int e = 0; e < 8; ++e) fin = fin && isfinite(a[e]) && isfinite(b[e]);
  if (!fin) record_status(status, (int)LSH_ERR_RANGE);
  if (wide) {
    // 32-byte aligned outputs: one 256-bit store per row piece, so every
    // store instruction writes whole sectors
    st_global_v8f(dv + t * 64 + c8, a);
    st_global_v8f(dqk + t * 64 + c8, b);
  } else {
    float4* pv = reinterpret_cast<float4*>(dv + t * 64 + c8);
    float4* pq = reinterpret_cast<float4*>(dqk + t * 64 + c8);
    pv[0] = make_float4(a[0], a[1], a[2], a[3]);
    pv[1] = make_float4(a[4], a[5], a[6], a[7]);
    pq[0] = make_float4(b[0], b[1], b[2], b[3]);
    pq[1] = make_float4(b[4], b[5], b[6], b[7]);
  }
}

bool tc_eligible(const lsh_problem& p) {
  if (p.dtype != LSH_BF16 || p.chunk != kM || !(p.scale > 0.f) || p.L % kM != 0) return false;
  const int n_pairs = (p.L / kM + 1) / 2;
  const int64_t units = (int64_t)p.B * p.H * p.n_rounds * ((n_pairs + kUnit - 1) / kUnit);
  const int64_t rows = (int64_t)p.B * p.H * p.n_rounds * p.L;
  return units <= INT32_MAX && rows <= INT32_MAX;
}

struct TcWs {
  __half* x16;
  __half* v16;
  __half* g16;
  int32_t* emap;
  __half* part_dv;
  __half* part_dqk;
  __half* edge;
  size_t bytes;
};
TcWs tc_ws(const lsh_problem& p, void* base) {
  const size_t rows = (size_t)p.B * p.H * p.n_rounds * p.L;
  const int n_pairs = (p.L / kM + 1) / 2;
  const size_t edge_rows =
      (size_t)p.B * p.H * p.n_rounds * ((n_pairs + kUnit - 1) / kUnit) * kM;
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  TcWs w;
  char* c = (char*)base;
  size_t off = 0;
  const size_t toks = (size_t)p.B * p.H * p.L;
  w.x16 = (__half*)(c + off);
  off += al(toks * 64 * 2);
  w.v16 = (__half*)(c + off);
  off += al(toks * 64 * 2);
  w.g16 = (__half*)(c + off);
  off += al(toks * 64 * 2);
  w.emap = (int32_t*)(c + off);
  off += al(rows * 4);
  w.part_dv = (__half*)(c + off);
  off += al(rows * 64 * 2);
  w.part_dqk = (__half*)(c + off);
  off += al(rows * 64 * 2);
  w.edge = (__half*)(c + off);
  off += al(edge_rows * 64 * 2);
  w.bytes = off;
  return w;
}

}  // namespace

size_t bwd_tc_ws_bytes(const lsh_problem& p) {
  return tc_eligible(p) ? tc_ws(p, nullptr).bytes : 0;
}

cudaError_t launch_attn_bwd_tc(const lsh_problem& p, const void* qk, const void* v,
                               const void* dout, const void* out, const void* out_lo,
                               const int32_t* perm, const float* lse, float* D, float* dqk,
                               float* dv, void* ws, int* status, cudaStream_t s) {
  if (!tc_eligible(p)) return cudaErrorNotSupported;
  const TcWs w = tc_ws(p, ws);
  const int n_chunks = p.L / kM;
  const int n_pairs = (n_chunks + 1) / 2;
  const int units_per_seg = (n_pairs + kUnit - 1) / kUnit;
  const int64_t n_segs = (int64_t)p.B * p.H * p.n_rounds;
  const int64_t n_units = n_segs * units_per_seg;
  const int64_t N = (int64_t)p.B * p.H * p.L;
  bwd_prep_tc_kernel<<<(unsigned)((N * 8 + 255) / 256), 256, 0, s>>>(
      (const __nv_bfloat16*)qk, (const __nv_bfloat16*)v, (const __nv_bfloat16*)dout,
      (const __nv_bfloat16*)out, (const __nv_bfloat16*)out_lo, D, w.x16, w.v16, w.g16, N);
  int grid = sm_count();
  if ((int64_t)grid > n_units) grid = (int)n_units;
  auto kern = p.causal ? attn_bwd_tc_kernel<true> : attn_bwd_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kSmemBytes, s>>>(
      w.x16, w.v16, w.g16, perm, lse, D,
      w.part_dv, w.part_dqk, w.edge, w.emap, p.L, p.n_rounds, p.scale, p.scale * kLog2e, (int)n_units,
      units_per_seg, status);
  sum_rounds_kernel<<<(unsigned)((N * 8 + 255) / 256), 256, 0, s>>>(
      w.part_dv, w.part_dqk, w.edge, w.emap, lse, (const __nv_bfloat16*)dout, dqk, dv, p.L,
      p.n_rounds, n_units * kM, N, (((uintptr_t)dqk | (uintptr_t)dv) & 31) == 0 ? 1 : 0, status);
  note_launch(3);
  return cudaGetLastError();
}

}  // namespace lsh
