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
//   warps 0-3  : producers — cp.async gathers of x and v rows through perm
//                (four whole 128-byte rows per instruction, eight lanes a row)
//                straight into the 128-byte-swizzled K-major layout of a
//                5-slot ring (a unit's first pair also needs chunk 2p0-1,
//                which goes to one of 3 rotating side buffers). v arrives
//                as an fp16 copy made before the launch (exact for
//                |values| < 65504); x stays bf16, whose products are exact
//                in the Q K^T MMA too. Software-pipelined one job deep, with
//                the next job's perm entries loaded a job ahead;
//   warp 12    : TMEM allocation; one elected lane issues S = Q K^T (three
//                128x64x64 MMAs per pair into a double-buffered TMEM S) and
//                O = P V with P read from TMEM (A operand) and V from shared
//                memory (MN-major B operand);
//   warps 4-7  : softmax warpgroup for even jobs, warps 8-11 for odd jobs —
//                one query row per thread, two passes over its 128 scores,
//                held in registers (the second 64-column TMEM load in flight
//                while the first block is masked): (1) causal/self mask and
//                row max; (2) exp2, row sum, P packed as fp16 pairs into TMEM
//                over S.
//                After publishing P, the warpgroup writes its previous job's
//                output: O from TMEM scaled by 1/l, as fp16, in original token
//                order (32-byte stores, whole sectors), + lse_r (so the stores
//                stay off the path from S to P).
// fp16 for P and V keeps P's rounding error at 2^-11 (bf16 would add about
// 3e-3 to O on the 64K workload).
#include <cuda_fp16.h>
#include <stddef.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"
#include "tma_host.h"

namespace lsh {
namespace {

using namespace tc;

constexpr int kM = 64;            // chunk
constexpr int kUnit = 8;          // pairs per work unit
constexpr int kSlots = 5;         // pair slots in the ring
constexpr int kPre = 3;           // side buffers for a unit's previous chunk
constexpr int kTile = 64 * 128;   // one chunk of 64 rows x 64 16-bit values = 8 KB
constexpr int kSlotBytes = 4 * kTile;   // x_even | x_odd | v_even | v_odd
constexpr int kPreBytes = 2 * kTile;    // x_prev | v_prev
constexpr int kThreads = 512;           // 4 warpgroups
// Register split (setmaxnreg): launched at 128 per thread (65536 / 512);
// producers and the MMA warpgroup drop to 56, the two softmax warpgroups
// rise to 200: 2*128*56 + 2*128*200 = 65536.
constexpr int kRegsLow = 64, kRegsHigh = 192;
static_assert(2 * 128 * kRegsLow + 2 * 128 * kRegsHigh <= kThreads * 128, "register split");
constexpr uint32_t kSCols = 192;        // TMEM columns of one S / P buffer
constexpr uint32_t kOCol = 2 * kSCols;  // first TMEM column of the O buffers

struct __align__(16) FwdBar {
  uint64_t slot_full[kSlots];
  uint64_t slot_free[kSlots];
  uint64_t pre_free[kPre];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t p_free[2];
  uint64_t o_free[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  // original positions of the slot's even|odd rows; read as int4, so
  // 16-byte aligned
  alignas(16) int kpos[kSlots][128];
  alignas(16) int kpos_pre[kPre][64];
};
static_assert(offsetof(FwdBar, kpos) % 16 == 0 && offsetof(FwdBar, kpos_pre) % 16 == 0,
              "position arrays are read with 16-byte loads");

constexpr size_t kSmemBytes = 1024 + kSlots * kSlotBytes + kPre * kPreBytes + sizeof(FwdBar);

struct Job {
  int64_t seg;   // (b*H + h)*n_rounds + r
  int p;         // pair index within the segment
  bool first;    // first pair of its unit
};

// Walks the CTA's units in order; every role iterates the same sequence.
struct JobIter {
  int unit, n_units, stride;
  int units_per_seg, n_pairs, k;
  __device__ JobIter(int u0, int nu, int st, int ups, int np)
      : unit(u0), n_units(nu), stride(st), units_per_seg(ups), n_pairs(np), k(0) {}
  __device__ bool next(Job& j) {
    while (unit < n_units) {
      const int seg = unit / units_per_seg;
      const int p = (unit - seg * units_per_seg) * kUnit + k;
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
// Packed float32 pairs: (a0, a1) * (b, b) + (c, c) and (a0, a1) + (b0, b1).
__device__ __forceinline__ float2 fma2(float a0, float a1, float b, float c) {
  uint64_t a, bb, cc, r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(bb) : "f"(b));
  asm("mov.b64 %0, {%1, %1};" : "=l"(cc) : "f"(c));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(bb), "l"(cc));
  float2 y;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(y.x), "=f"(y.y) : "l"(r));
  return y;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  uint64_t x, y, r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(y) : "f"(b.x), "f"(b.y));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(x), "l"(y));
  float2 z;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(z.x), "=f"(z.y) : "l"(r));
  return z;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// One 32-byte store (the address is 32-byte aligned).
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]),
               "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

// Warp w copies rows 16 w .. 16 w + 15 of a chunk tile into their
// 128-byte-swizzled places, four whole rows per instruction (eight lanes per
// row, one 16-byte piece each). Lane j (and j + 16) holds the position of
// row 16 w + j; called by the whole warp.
template <typename T16>
__device__ __forceinline__ void issue_rows(const T16* __restrict__ src, uint8_t* tile, int pos,
                                           int w, int lane) {
  const uint32_t base = smem_u32(tile);
  const int rsub = lane >> 3, ch = lane & 7;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int r = 16 * w + 4 * g + rsub;
    const int ps = __shfl_sync(0xffffffffu, pos, 4 * g + rsub);
    cp_async16(base + r * 128 + (((uint32_t)ch ^ (uint32_t)(r & 7)) << 4),
               src + (int64_t)ps * 64 + ch * 8);
  }
}

// ---- MMA issue helpers (one thread); descriptor lower words are shared
// addresses >> 4 plus the LBO field of the operand layout.
constexpr uint32_t kIdS64 = idesc_f16(128, 64, 1, false, false);    // Q K^T: bf16, K-major
constexpr uint32_t kIdS128 = idesc_f16(128, 128, 1, false, false);
constexpr uint32_t kIdO = idesc_f16(128, 64, 0, false, true);       // P V: fp16, V MN-major
constexpr uint32_t kLboK = desc_lbo(16), kLboV = desc_lbo(kTile);

// S = Q K^T of job nn (slot nn % kSlots, TMEM buffer nn & 1): key block 0 is
// the previous chunk (side buffer pb, or the previous slot's odd chunk);
// blocks 1 and 2 (this slot's chunks, contiguous) go in one N = 128 product.
__device__ __forceinline__ bool fwd_issue_s(FwdBar* bar, uint32_t tmem, uint32_t slot0,
                                            uint32_t pre0, const Job& jb, int nn, int pb,
                                            int n_chunks, volatile int* abort, int* status) {
  const int s = nn % kSlots, b = nn & 1;
  if (!__all_sync(0xffffffffu, mbar_wait(&bar->slot_full[s], (uint32_t)(nn / kSlots) & 1u, abort, status))) return false;
  tc_fence_after();
  const uint32_t sl = slot0 + (uint32_t)(s * kSlotBytes) / 16;
  const uint32_t d = tmem + (uint32_t)b * kSCols;
  const bool has_prev = jb.p > 0, has_odd = 2 * jb.p + 1 < n_chunks;
  const uint32_t q = sl + kLboK;
  const uint32_t prev_x = pb >= 0 ? pre0 + (uint32_t)(pb * kPreBytes) / 16
                                  : slot0 + (uint32_t)(((nn + kSlots - 1) % kSlots) * kSlotBytes + kTile) / 16;
  const uint32_t id_main = has_odd ? kIdS128 : kIdS64;
  if (elect_one()) {
    if (has_prev) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_ss_raw(d, q + 2 * ks, prev_x + kLboK + 2 * ks, kDescHi1024, kIdS64, ks > 0);
    }
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
      mma_ss_raw(d + 64, q + 2 * ks, q + 2 * ks, kDescHi1024, id_main, ks > 0);
    mma_commit_raw(&bar->s_full[b]);
  }
  __syncwarp();
  return true;
}
// O (+)= P[:, 64 keys] V_block with P from TMEM; issued by the calling
// (elected) thread.
__device__ __forceinline__ void fwd_issue_pv(uint32_t d, uint32_t pa, uint32_t v_lo, bool acc) {
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
    mma_ts_raw(d, pa + ks * 8, v_lo + 128 * ks, kDescHi1024, kIdO, acc || ks > 0);
}

template <bool kCausal>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_tc_kernel(const __nv_bfloat16* __restrict__ qk, const __half* __restrict__ v,
                   const int32_t* __restrict__ perm, __half* __restrict__ opart,
                   float* __restrict__ lsepart, int L, int n_rounds, int64_t N, float scale_log2,
                   int n_units, int units_per_seg, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* slots = smem;
  uint8_t* pres = slots + kSlots * kSlotBytes;
  FwdBar* bar = (FwdBar*)(pres + kPre * kPreBytes);
  volatile int* abort = &bar->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_chunks = L / kM;
  const int n_pairs = (n_chunks + 1) / 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&bar->slot_full[s], 128);
      mbar_init(&bar->slot_free[s], 1);
    }
    for (int s = 0; s < kPre; ++s) mbar_init(&bar->pre_free[s], 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar->s_full[b], 1);
      mbar_init(&bar->p_full[b], 128);
      mbar_init(&bar->p_free[b], 1);
      mbar_init(&bar->o_free[b], 128);
    }
    mbar_init(&bar->mma_done, 1);
    bar->abort = 0;
    fence_mbar_init();
  }
  if (warp == 12) {
    tmem_alloc(&bar->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  const int wgi = warp >> 2;

  if (wgi == 0) {
    // ------------------------------------------------ producers
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
    // lane j and j + 16 of warp w hold the positions of row 16 w + j
    const int row = 16 * warp + (lane & 15);
    JobIter it(blockIdx.x, n_units, gridDim.x, units_per_seg, n_pairs);
    Job cur, nxt;
    bool have_cur = it.next(cur);
    // perm entries of the next job are loaded one iteration ahead and only
    // checked when used, so the loads overlap the rest of the iteration
    int pos_p = 0, pos_e = 0, pos_o = 0;
    auto fetch_pos = [&](const Job& jb) {
      const int32_t* pr = perm + jb.seg * L + row;
      pos_e = __ldg(pr + (int64_t)(2 * jb.p) * kM);
      pos_o = (2 * jb.p + 1 < n_chunks) ? __ldg(pr + (int64_t)(2 * jb.p + 1) * kM) : 0;
      pos_p = (jb.first && jb.p > 0) ? __ldg(pr + (int64_t)(2 * jb.p - 1) * kM) : 0;
    };
    auto checked = [&](int ps) {
      if ((unsigned)ps >= (unsigned)L) {
        record_status(status, (int)LSH_ERR_DEVICE_CHECK);
        ps = 0;
      }
      return ps;
    };
    if (have_cur) fetch_pos(cur);
    int n = 0, pre_uses = 0;
    bool pend = false, pend_odd = false;
    int pend_slot = 0, pend_pre = -1;
    bool ok = true;
    auto publish = [&]() {
      fence_proxy_async();
      mbar_arrive(&bar->slot_full[pend_slot]);
    };
    while (have_cur) {
      const int s = n % kSlots;
      if (n >= kSlots &&
          !mbar_wait(&bar->slot_free[s], (uint32_t)(n / kSlots - 1) & 1u, abort, status)) {
        ok = false;
        break;
      }
      const bool use_pre = cur.first && cur.p > 0, has_odd = 2 * cur.p + 1 < n_chunks;
      int pb_idx = -1;
      if (use_pre) {
        pb_idx = pre_uses % kPre;
        if (pre_uses >= kPre &&
            !mbar_wait(&bar->pre_free[pb_idx], (uint32_t)(pre_uses / kPre - 1) & 1u, abort,
                       status)) {
          ok = false;
          break;
        }
        ++pre_uses;
      }
      const int64_t bh = cur.seg / n_rounds;
      pos_e = checked(pos_e);
      pos_o = checked(pos_o);
      pos_p = checked(pos_p);
      uint8_t* sl = slots + s * kSlotBytes;
      const __nv_bfloat16* xb = qk + bh * L * 64;
      const __half* vb = v + bh * L * 64;
      if (use_pre) {
        uint8_t* pb = pres + pb_idx * kPreBytes;
        if (lane < 16) bar->kpos_pre[pb_idx][row] = pos_p;
        issue_rows(xb, pb, pos_p, warp, lane);
        issue_rows(vb, pb + kTile, pos_p, warp, lane);
      }
      if (lane < 16) bar->kpos[s][row] = pos_e;
      issue_rows(xb, sl, pos_e, warp, lane);
      issue_rows(vb, sl + 2 * kTile, pos_e, warp, lane);
      if (has_odd) {
        if (lane < 16) bar->kpos[s][64 + row] = pos_o;
        issue_rows(xb, sl + kTile, pos_o, warp, lane);
        issue_rows(vb, sl + 3 * kTile, pos_o, warp, lane);
      }
      cp_async_commit();
      have_cur = it.next(nxt);
      if (have_cur) fetch_pos(nxt);
      if (pend) {
        cp_async_wait<1>();
        publish();
      }
      pend = true;
      pend_slot = s;
      pend_pre = pb_idx;
      pend_odd = has_odd;
      cur = nxt;
      ++n;
    }
    cp_async_wait<0>();
    if (pend && ok) publish();
  } else if (wgi == 3) {
    // ------------------------------------------------ MMA issuer (warp 12)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
    if (warp == 12) {
      const uint32_t slot0 = smem_u32(slots) >> 4, pre0 = smem_u32(pres) >> 4;
      JobIter it(blockIdx.x, n_units, gridDim.x, units_per_seg, n_pairs);
      Job cur, nxt;
      bool have_cur = it.next(cur);
      int n = 0, pre_uses = 0;
      int cur_pre = -1, nxt_pre = -1;
      bool ok = true;
      if (have_cur) {
        if (cur.first && cur.p > 0) cur_pre = pre_uses++ % kPre;
        ok = fwd_issue_s(bar, tmem, slot0, pre0, cur, 0, cur_pre, n_chunks, abort, status);
      }
      while (have_cur && ok) {
        const bool have_nxt = it.next(nxt);
        nxt_pre = -1;
        if (have_nxt && nxt.first && nxt.p > 0) nxt_pre = pre_uses++ % kPre;
        if (have_nxt && !fwd_issue_s(bar, tmem, slot0, pre0, nxt, n + 1, nxt_pre, n_chunks, abort, status))
          break;
        // O = P V for job n
        const int b = n & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&bar->p_full[b], (uint32_t)(n / 2) & 1u, abort, status))) break;
        if (n >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bar->o_free[b], (uint32_t)(n / 2 - 1) & 1u, abort, status)))
          break;
        tc_fence_after();
        const int s = n % kSlots;
        const uint32_t sl = slot0 + (uint32_t)(s * kSlotBytes) / 16;
        const bool has_prev = cur.p > 0, has_odd = 2 * cur.p + 1 < n_chunks;
        const uint32_t prev_v =
            cur_pre >= 0 ? pre0 + (uint32_t)(cur_pre * kPreBytes + kTile) / 16
                         : slot0 + (uint32_t)(((n + kSlots - 1) % kSlots) * kSlotBytes + 3 * kTile) / 16;
        const uint32_t d = tmem + kOCol + (uint32_t)b * 64;
        const uint32_t pa = tmem + (uint32_t)b * kSCols;
        // key block 0 (previous chunk) when present, then blocks 1 and 2
        if (elect_one()) {
          if (has_prev) fwd_issue_pv(d, pa, prev_v + kLboV, false);
          fwd_issue_pv(d, pa + 32, sl + 2 * kTile / 16 + kLboV, has_prev);
          if (has_odd) fwd_issue_pv(d, pa + 64, sl + 3 * kTile / 16 + kLboV, true);
          mma_commit_raw(&bar->p_free[b]);                // P(n) consumed, O(n) ready
          if (n >= 1) mma_commit_raw(&bar->slot_free[(n - 1) % kSlots]);
          if (cur_pre >= 0) mma_commit_raw(&bar->pre_free[cur_pre]);
        }
        __syncwarp();
        cur = nxt;
        cur_pre = nxt_pre;
        have_cur = have_nxt;
        ++n;
      }
      mma_commit(&bar->mma_done);
      int dummy = 0;
      mbar_wait(&bar->mma_done, 0, (volatile int*)&dummy, status);
    }
  } else {
    // ------------------------------------------------ softmax warpgroups
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
    const int wg = wgi - 1;                     // 0: even jobs, 1: odd jobs
    const int q = warp & 3;                     // TMEM lane quarter (rows 32q..32q+31)
    const int row = q * 32 + lane;              // query row in the pair tile
    const bool odd_row = row >= 64;             // row belongs to chunk 2p+1
    const int kb0 = odd_row ? 1 : 0;            // first key block of this row
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t sbuf = tmem + lane_off + (uint32_t)wg * kSCols;
    const uint32_t obuf = tmem + lane_off + kOCol + (uint32_t)wg * 64;
    JobIter it(blockIdx.x, n_units, gridDim.x, units_per_seg, n_pairs);
    Job j;
    int n = 0, pre_uses = 0;
    bool pend = false, pend_write = false;
    float pend_inv_l = 0.f, pend_lse = 0.f;
    int64_t pend_row = 0;
    int pend_n = 0;
    auto epilogue = [&]() {
      // O of this warpgroup's previous job is complete once its PV is done
      if (!mbar_wait(&bar->p_free[wg], (uint32_t)(pend_n / 2) & 1u, abort, status)) return false;
      tc_fence_after();
      uint4* dst = reinterpret_cast<uint4*>(opart + pend_row * 64);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t o[32];
        tmem_ld32(obuf + 32 * h, o);
        tmem_ld_wait();
        if (h == 1) {
          tc_fence_before();
          mbar_arrive(&bar->o_free[wg]);
        }
        if (pend_write) {
          // whole 32-byte sectors: 16 columns per 256-bit store
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t w[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
              w[k] = pack_f16x2(__uint_as_float(o[16 * c + 2 * k]) * pend_inv_l,
                                __uint_as_float(o[16 * c + 2 * k + 1]) * pend_inv_l);
            st_global_v8(dst + 4 * h + 2 * c, w);
          }
        }
      }
      if (pend_write) lsepart[pend_row] = pend_lse;
      return true;
    };
    bool ok = true;
    while (ok && it.next(j)) {
      const bool use_pre = j.first && j.p > 0;
      const int pb = use_pre ? pre_uses++ % kPre : -1;
      if ((n & 1) != wg) { ++n; continue; }
      const int s = n % kSlots;
      if (!mbar_wait(&bar->s_full[wg], (uint32_t)(n / 2) & 1u, abort, status)) break;
      tc_fence_after();
      const bool has_prev = j.p > 0, has_odd = 2 * j.p + 1 < n_chunks;
      const bool row_live = !odd_row || has_odd;
      const int qpos = bar->kpos[s][row];
      const int* kp_lo = kb0 == 0 ? (pb >= 0 ? bar->kpos_pre[pb]
                                             : bar->kpos[(n + kSlots - 1) % kSlots] + 64)
                                  : bar->kpos[s];
      const int* kp_hi = kb0 == 0 ? bar->kpos[s] : bar->kpos[s] + 64;
      const bool lo_ok = kb0 == 0 ? has_prev : true;
      // pass 1: mask and row max over this row's 128 keys; masked values
      // (-inf) are written back so pass 2 needs no positions. Two TMEM loads
      // per wait and four independent max chains keep latency off the path.
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      // the second 64-column block's TMEM load is in flight while the first
      // one is masked (and, in pass 2, exponentiated)
      uint32_t sv[2][64];
      const uint32_t col0 = (uint32_t)(kb0 * 64), col1 = col0 + 64;
      tmem_ld32(sbuf + col0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0][0]));
      tmem_ld32(sbuf + col0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[0][32]));
      tmem_ld_wait();
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        if (c2 == 0) {
          tmem_ld32(sbuf + col1, *reinterpret_cast<uint32_t(*)[32]>(&sv[1][0]));
          tmem_ld32(sbuf + col1 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[1][32]));
        }
        const uint32_t col = c2 ? col1 : col0;
        const int* kp = (c2 == 0) ? kp_lo : kp_hi;
        const bool blk_ok = (c2 == 0) ? lo_ok : true;
#pragma unroll
        for (int i4 = 0; i4 < 16; ++i4) {
          const int4 k4 = blk_ok ? *reinterpret_cast<const int4*>(kp + 4 * i4)
                                 : make_int4(0, 0, 0, 0);
          const int kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = 4 * i4 + e;
            const bool valid = blk_ok && (kCausal ? (kk[e] < qpos) : (kk[e] != qpos));
            sv[c2][i] = valid ? sv[c2][i] : __float_as_uint(-INFINITY);
          }
          // two 3-input maxima per four scores
          mx4[i4 & 3] = max3(mx4[i4 & 3], __uint_as_float(sv[c2][4 * i4]),
                             __uint_as_float(sv[c2][4 * i4 + 1]));
          mx4[(i4 + 2) & 3] = max3(mx4[(i4 + 2) & 3], __uint_as_float(sv[c2][4 * i4 + 2]),
                                   __uint_as_float(sv[c2][4 * i4 + 3]));
        }
        (void)col;
        if (c2 == 0) tmem_ld_wait();
      }
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      const bool has = mx != -INFINITY;
      const float neg = has ? -mx * scale_log2 : 0.f;
      // pass 2: P = exp2(scale * (s - max)) as fp16 pairs into TMEM over S;
      // P column block kb lives at TMEM columns [32 kb, 32 kb + 32). The masked
      // values are still in registers, so nothing is read back.
      float2 l2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float2 t = fma2(__uint_as_float(sv[c2][2 * e]), __uint_as_float(sv[c2][2 * e + 1]),
                                scale_log2, neg);
          const float2 p2 = make_float2(ex2(t.x), ex2(t.y));
          l2[e & 1] = add2(l2[e & 1], p2);
          pk[e] = pack_f16x2(p2.x, p2.y);
        }
        tmem_st16(sbuf + (uint32_t)(kb0 * 32 + c2 * 32), *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
        tmem_st16(sbuf + (uint32_t)(kb0 * 32 + c2 * 32 + 16), *reinterpret_cast<uint32_t(*)[16]>(&pk[16]));
      }
      const float l = (l2[0].x + l2[0].y) + (l2[1].x + l2[1].y);
      {
        uint32_t z[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) z[e] = 0u;
        tmem_st32(sbuf + (uint32_t)(odd_row ? 0 : 64), z);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bar->p_full[wg]);
      // the previous job's output is written now, off the path from S to P
      // (this job's PV waits only for its TMEM read, signalled by o_free)
      if (pend && !epilogue()) break;
      pend = true;
      pend_n = n;
      pend_write = row_live;
      const int64_t bh = j.seg / n_rounds;
      const int r = (int)(j.seg % n_rounds);
      pend_row = (int64_t)r * N + bh * L + qpos;
      pend_inv_l = has ? 1.f / l : 0.f;
      pend_lse = has ? (mx * scale_log2 + log2f(l)) * kLn2 : -INFINITY;
      ++n;
    }
    if (pend && !*abort) epilogue();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool launch_attn_fwd_tc_ok(const lsh_problem& p) {
  if (p.dtype != LSH_BF16 || p.chunk != kM || !(p.scale > 0.f)) return false;
  const int64_t n_units =
      (int64_t)p.B * p.H * p.n_rounds * (((p.L / kM + 1) / 2 + kUnit - 1) / kUnit);
  return n_units <= INT32_MAX;
}

cudaError_t launch_attn_fwd_tc(const lsh_problem& p, const void* qk, const void* v,
                               const int32_t* perm, void* opart_f16, float* lsepart, int* status,
                               cudaStream_t s) {
  if (!launch_attn_fwd_tc_ok(p)) return cudaErrorNotSupported;
  const int n_chunks = p.L / kM;
  const int n_pairs = (n_chunks + 1) / 2;
  const int units_per_seg = (n_pairs + kUnit - 1) / kUnit;
  const int64_t n_segs = (int64_t)p.B * p.H * p.n_rounds;
  const int64_t n_units = n_segs * units_per_seg;
  const int64_t N = (int64_t)p.B * p.H * p.L;
  if (n_units > INT32_MAX) return cudaErrorNotSupported;
  int grid = sm_count();
  if ((int64_t)grid > n_units) grid = (int)n_units;
  auto kern = p.causal ? attn_fwd_tc_kernel<true> : attn_fwd_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kSmemBytes, s>>>((const __nv_bfloat16*)qk, (const __half*)v, perm,
                                          (__half*)opart_f16, lsepart, p.L, p.n_rounds, N,
                                          p.scale * kLog2e, (int)n_units, units_per_seg, status);
  note_launch();
  return cudaGetLastError();
}

}  // namespace lsh
