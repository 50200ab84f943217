// LSH bucket assignment on the 5th-generation tensor cores (bf16 inputs).
//
// "Reformer: The Efficient Transformer" (research.elamur.ai summary page),
// Key points, "LSH attention": h(x) = argmax([xR; -xR]). Column k of x R_r
// appears as +s_k (index k) and -s_k (index n_b/2 + k), so the argmax is the
// column with the largest |s_k|, moved to the second half when s_k < 0.
//
// bf16 x and bf16 R multiply exactly in float32, and the tensor core adds the
// products into float32 accumulators in TMEM: this is a float32 contraction
// of exact products, as on the CUDA-core path.
//
// Structure (one CTA per SM, persistent; CTAs are assigned to one round so
// that R_r stays resident in shared memory):
//   warp 0  : TMA producer — R_r once (MN-major operand), then 128-token X
//             tiles (K-major) through a 4-stage ring, released by the MMAs;
//   warp 1  : TMEM allocation; one thread issues tcgen05.mma: a 128 x 256 x 64
//             product per 256-column chunk of R_r;
//   warps 2-5, 6-9: two epilogue warpgroups taking alternate tiles, each with
//             its own 256-column TMEM accumulator (one token per thread).
//             Each s becomes a float key whose 4 low mantissa bits hold
//             (15 - its 32-column group) and whose sign is kept; two 3-input
//             max and min operations fold two columns into each of 32
//             per-position running maxima (largest +s) and minima (most
//             negative s), the lowest column winning ties. Values closer than
//             2^-19 relative count as ties (a near-tie by the 1e-5 bound the
//             results are checked against). The merge picks the larger of the
//             best +s and the best -s, the +s half first on ties.
// Handles n_b/2 <= 512 with n_b/2 a multiple of 8; other shapes use the
// CUDA-core kernel.
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"
#include "tma_host.h"

namespace lsh {
namespace {

using namespace tc;

constexpr int kTileM = 128;          // tokens per tile
constexpr int kStages = 4;           // X ring depth
constexpr int kMaxNh = 512;          // rotation columns resident per round
constexpr int kChunkN = 256;         // columns per MMA / accumulator
constexpr int kXBytes = kTileM * 128;              // 16 KB
constexpr int kRBlockBytes = 64 * 128;             // 64 columns x 64 k-rows
constexpr int kRBytes = (kMaxNh / 64) * kRBlockBytes;  // 64 KB
constexpr int kThreads = 320;

struct __align__(8) HashBarriers {
  uint64_t r_full;
  uint64_t x_full[kStages];
  uint64_t x_empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kSmemBytes = 1024 + kRBytes + kStages * kXBytes + sizeof(HashBarriers);

__device__ __forceinline__ bool warp_all(bool ok) { return __all_sync(0xffffffffu, ok); }

// Folds two accumulator values (raw fp32 bits a, b; group tags ta, tb in the
// low 4 mantissa bits) into the running maximum and minimum of one position.
__device__ __forceinline__ void fold2(float& mx, float& mn, uint32_t a, uint32_t b, uint32_t ta,
                                      uint32_t tb) {
  const float ka = __uint_as_float((a & 0xFFFFFFF0u) | ta);
  const float kb = __uint_as_float((b & 0xFFFFFFF0u) | tb);
  float r0, r1;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r0) : "f"(mx), "f"(ka), "f"(kb));
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r1) : "f"(mn), "f"(ka), "f"(kb));
  mx = r0;
  mn = r1;
}

__global__ void __launch_bounds__(kThreads, 1)
hash_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_r,
               int32_t* __restrict__ bucket, int64_t n_rows, int L, int nh, int n_rounds,
               int n_tiles, int ctas_per_round, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* r_smem = smem;
  uint8_t* x_smem = smem + kRBytes;
  HashBarriers* bar = (HashBarriers*)(x_smem + kStages * kXBytes);
  volatile int* abort = &bar->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x % n_rounds;
  const int ci = blockIdx.x / n_rounds;
  const int n_blk = (nh + 63) / 64;
  const int nsub = (nh + kChunkN - 1) / kChunkN;

  if (threadIdx.x == 0) {
    mbar_init(&bar->r_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar->x_full[s], 1);
      mbar_init(&bar->x_empty[s], 1);     // released by the MMAs' commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar->acc_full[b], 1);
      mbar_init(&bar->acc_empty[b], 128);
    }
    mbar_init(&bar->mma_done, 1);
    bar->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- producer ----------------
      prefetch_tmap(&map_x);
      prefetch_tmap(&map_r);
      mbar_expect_tx(&bar->r_full, n_blk * kRBlockBytes);
      for (int b = 0; b < n_blk; ++b)
        tma_load_2d(r_smem + b * kRBlockBytes, &map_r, b * 64, r * 64, &bar->r_full);
      int it = 0;
      for (int t = ci; t < n_tiles; t += ctas_per_round, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (uint32_t)(it / kStages) & 1u;
        if (it >= kStages && !mbar_wait(&bar->x_empty[s], ph ^ 1u, abort, status)) break;
        mbar_expect_tx(&bar->x_full[s], kXBytes);
        tma_load_2d(x_smem + s * kXBytes, &map_x, 0, t * kTileM, &bar->x_full[s]);
      }
      // every issued copy has landed before the CTA may exit (bounded)
      const int issued = it;
      for (int s = 0; s < kStages && s < issued; ++s) {
        const int last = issued - 1 - ((issued - 1 - s) % kStages);
        int dummy = 0;
        mbar_wait(&bar->x_full[s], (uint32_t)(last / kStages) & 1u, (volatile int*)&dummy, status);
      }
      int dummy = 0;
      mbar_wait(&bar->r_full, 0, (volatile int*)&dummy, status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      // Tiles alternate between the two accumulators / epilogue warpgroups;
      // the chunks of a pair of tiles are interleaved so both stay busy.
      if (mbar_wait(&bar->r_full, 0, abort, status)) {
        tc_fence_after();
        const uint32_t r_lo = (smem_u32(r_smem) >> 4) | desc_lbo(kRBlockBytes);
        const uint32_t x_lo = (smem_u32(x_smem) >> 4) | desc_lbo(16);
        int uses0 = 0, uses1 = 0;
        bool ok = true;
        const int n_mine = (n_tiles - ci + ctas_per_round - 1) / ctas_per_round;
        for (int it0 = 0; it0 < n_mine && ok; it0 += 2) {
          const int cnt = min(2, n_mine - it0);
          for (int k = 0; k < cnt && ok; ++k)
            ok = mbar_wait(&bar->x_full[(it0 + k) % kStages],
                           (uint32_t)((it0 + k) / kStages) & 1u, abort, status);
          if (!ok) break;
          tc_fence_after();
          for (int j = 0; j < nsub && ok; ++j)
            for (int k = 0; k < cnt && ok; ++k) {
              const int it = it0 + k, w = it & 1, s = it % kStages;
              int& uses = w ? uses1 : uses0;
              if (uses > 0 &&
                  !mbar_wait(&bar->acc_empty[w], (uint32_t)(uses - 1) & 1u, abort, status)) {
                ok = false;
                break;
              }
              ++uses;
              tc_fence_after();
              const int ncols = min(kChunkN, nh - j * kChunkN);
              // whole 64-column blocks: the MN-major operand is read in complete
              // swizzle atoms; the zero-filled extra columns are masked later
              const int n_mma = (ncols + 63) / 64 * 64;
              const uint32_t idesc = idesc_f16(kTileM, n_mma, 1, false, true);
              const uint32_t d = tmem + (uint32_t)(w * kChunkN);
              const uint32_t a = x_lo + (uint32_t)(s * kXBytes) / 16;
              const uint32_t b = r_lo + (uint32_t)(j * 4 * kRBlockBytes) / 16;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_ss_w(d, a + 2 * kk, b + 128 * kk, kDescHi1024, idesc, kk > 0);
              mma_commit(&bar->acc_full[w]);
              if (j == nsub - 1) mma_commit(&bar->x_empty[s]);
            }
        }
      }
      // all issued MMAs have finished before TMEM is released (bounded)
      mma_commit(&bar->mma_done);
      int dummy = 0;
      mbar_wait(&bar->mma_done, 0, (volatile int*)&dummy, status);
    }
  } else {
    // ---------------- epilogue: warps 2..5 and 6..9 ----------------
    const int w = (warp - 2) >> 2;          // warpgroup = accumulator = tile parity
    const int q = warp & 3;                 // TMEM lane quarter this warp may read
    const int row_in_tile = q * 32 + lane;
    const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(w * kChunkN);
    int use = 0, it = 0;
    bool ok = true;
    for (int t = ci; t < n_tiles && ok; t += ctas_per_round, ++it) {
      if ((it & 1) != w) continue;
      float mx[32], mn[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        mx[i] = -INFINITY;
        mn[i] = INFINITY;
      }
      int g = 0;                              // global 32-column group index
      for (int j = 0; j < nsub; ++j, ++use) {
        if (!warp_all(mbar_wait(&bar->acc_full[w], (uint32_t)use & 1u, abort, status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int ncols = min(kChunkN, nh - j * kChunkN);
        for (int c0 = 0; c0 < ncols; c0 += 64, g += 2) {
          uint32_t va[32], vb[32];
          tmem_ld32(tbase + c0, va);
          tmem_ld32(tbase + c0 + 32, vb);     // within the accumulator's 256 columns
          tmem_ld_wait();
          const uint32_t ma = (uint32_t)(15 - g), mb = (uint32_t)(14 - g);
          if (ncols - c0 >= 64) {
#pragma unroll
            for (int i = 0; i < 32; ++i) fold2(mx[i], mn[i], va[i], vb[i], ma, mb);
          } else {
            const int na = ncols - c0, nb = ncols - c0 - 32;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              // a missing column is a NaN key, which max and min ignore
              const uint32_t a = (i < na) ? va[i] : 0x7FFFFFFFu;
              const uint32_t b = (i < nb) ? vb[i] : 0x7FFFFFFFu;
              fold2(mx[i], mn[i], a, b, ma, mb);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&bar->acc_empty[w]);
      }
      if (!ok) break;
      // merge: largest |s| over both halves; on ties the +s half, then the
      // smaller column
      uint32_t best_m = 0;
      int best_c = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const uint32_t kp = __float_as_uint(mx[i]), kn = __float_as_uint(mn[i]);
        // a negative running maximum or a positive running minimum (this
        // includes the initial -inf / +inf) is never the winner
        const bool vp = (kp >> 31) == 0u, vq = (kn >> 31) != 0u;
        const uint32_t mp = vp ? (kp & 0x7FFFFFF0u) : 0u;
        const int cp = vp ? (15 - (int)(kp & 15u)) * 32 + i : 0x7fffffff;
        const uint32_t mq = vq ? (kn & 0x7FFFFFF0u) : 0u;
        const int cq = vq ? nh + (15 - (int)(kn & 15u)) * 32 + i : 0x7fffffff;
        if (mp > best_m || (mp == best_m && cp < best_c)) { best_m = mp; best_c = cp; }
        if (mq > best_m || (mq == best_m && cq < best_c)) { best_m = mq; best_c = cq; }
      }
      const int64_t row = (int64_t)t * kTileM + row_in_tile;
      if (row < n_rows) {
        const int64_t bh = row / L, pos = row - bh * L;
        bucket[(bh * n_rounds + r) * L + pos] = best_c;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_hash_tc(const lsh_problem& p, const void* qk, const void* R, int32_t* bucket,
                           int* status, cudaStream_t s) {
  const int nh = p.n_buckets / 2;
  if (p.dtype != LSH_BF16 || nh > kMaxNh || nh % 8 != 0 || ((uintptr_t)R % 16) != 0)
    return cudaErrorNotSupported;
  const int64_t n_rows = (int64_t)p.B * p.H * p.L;
  const int64_t n_tiles64 = (n_rows + kTileM - 1) / kTileM;
  if (n_tiles64 > INT32_MAX) return cudaErrorNotSupported;
  const int n_tiles = (int)n_tiles64;
  CUtensorMap map_x, map_r;
  if (!encode_tmap_2d_16bit(&map_x, qk, 64, (uint64_t)n_rows, 128, 64, kTileM))
    return cudaErrorNotSupported;
  if (!encode_tmap_2d_16bit(&map_r, R, (uint64_t)nh, (uint64_t)p.n_rounds * 64,
                            (uint64_t)nh * 2, 64, 64))
    return cudaErrorNotSupported;
  int cpr = sm_count() / p.n_rounds;
  if (cpr < 1) cpr = 1;
  if (cpr > n_tiles) cpr = n_tiles;
  const int grid = cpr * p.n_rounds;
  cudaError_t e = cudaFuncSetAttribute(hash_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  hash_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(map_x, map_r, bucket, n_rows, p.L, nh,
                                                   p.n_rounds, n_tiles, cpr, status);
  note_launch();
  return cudaGetLastError();
}

}  // namespace lsh
