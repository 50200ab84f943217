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
//             tiles (K-major) through a 4-stage ring;
//   warp 1  : TMEM allocation; one thread issues tcgen05.mma: a 128 x N x 64
//             product per 256-column chunk of R_r into one of two TMEM
//             accumulators (so the epilogue of one chunk overlaps the MMA of
//             the next);
//   warps 2-5: epilogue — tcgen05.ld of the accumulator rows (one token per
//             thread). Each |s| becomes a float key whose 4 low mantissa bits
//             hold (15 - its 32-column group), so one 3-input max folds two
//             columns into each of 32 per-position running maxima with the
//             lowest column winning ties; values closer than 2^-19 relative
//             count as ties (a near-tie by the 1e-5 bound the results are
//             checked against). The winner's sign is recomputed from the X and
//             R tiles in shared memory, then the bucket id is written.
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
constexpr int kThreads = 192;

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
      mbar_init(&bar->x_empty[s], 128);   // released by the epilogue (sign recompute)
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
      if (mbar_wait(&bar->r_full, 0, abort, status)) {
        tc_fence_after();
        const uint32_t r_base = smem_u32(r_smem);
        const uint32_t x_base = smem_u32(x_smem);
        int it = 0, job = 0;
        bool ok = true;
        for (int t = ci; t < n_tiles && ok; t += ctas_per_round, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&bar->x_full[s], (uint32_t)(it / kStages) & 1u, abort, status)) break;
          tc_fence_after();
          for (int j = 0; j < nsub; ++j, ++job) {
            const int buf = job & 1;
            const int use = job >> 1;
            if (use > 0 && !mbar_wait(&bar->acc_empty[buf], (uint32_t)(use - 1) & 1u, abort, status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const int ncols = min(kChunkN, nh - j * kChunkN);
            // whole 64-column blocks: the MN-major operand is read in complete
            // swizzle atoms; the zero-filled extra columns are masked later
            const int n_mma = (ncols + 63) / 64 * 64;
            const uint32_t idesc = idesc_f16(kTileM, n_mma, 1, false, true);
            const uint32_t d = tmem + (uint32_t)(buf * kChunkN);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              uint64_t a = smem_desc(x_base + s * kXBytes + k * 32, 16, 1024);
              uint64_t b = smem_desc(r_base + j * 4 * kRBlockBytes + k * 2048, kRBlockBytes, 1024);
              mma_ss(d, a, b, idesc, k > 0 ? 1u : 0u);
            }
            mma_commit(&bar->acc_full[buf]);
          }
        }
      }
      // all issued MMAs have finished before TMEM is released (bounded)
      mma_commit(&bar->mma_done);
      int dummy = 0;
      mbar_wait(&bar->mma_done, 0, (volatile int*)&dummy, status);
    }
  } else {
    // ---------------- epilogue: warps 2..5 ----------------
    const int q = warp & 3;                 // TMEM lane quarter this warp may read
    const int row_in_tile = q * 32 + lane;
    int job = 0, it = 0;
    bool ok = true;
    for (int t = ci; t < n_tiles && ok; t += ctas_per_round, ++it) {
      float acc[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) acc[i] = 0.f;
      int g = 0;                              // global 32-column group index
      for (int j = 0; j < nsub; ++j, ++job) {
        const int buf = job & 1;
        if (!mbar_wait(&bar->acc_full[buf], (uint32_t)(job >> 1) & 1u, abort, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int ncols = min(kChunkN, nh - j * kChunkN);
        const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * kChunkN);
        for (int c0 = 0; c0 < ncols; c0 += 64, g += 2) {
          uint32_t va[32], vb[32];
          tmem_ld32(taddr + c0, va);
          tmem_ld32(taddr + c0 + 32, vb);     // within the 512 allocated columns
          tmem_ld_wait();
          const uint32_t ma = (uint32_t)(15 - g), mb = (uint32_t)(14 - g);
          const int na = min(32, ncols - c0), nb = min(32, ncols - c0 - 32);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const uint32_t ka = (i < na) ? ((va[i] & 0x7FFFFFF0u) | ma) : 0u;
            const uint32_t kb = (i < nb) ? ((vb[i] & 0x7FFFFFF0u) | mb) : 0u;
            float r;
            asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(acc[i]), "f"(__uint_as_float(ka)),
                "f"(__uint_as_float(kb)));
            acc[i] = r;
          }
        }
        tc_fence_before();
        mbar_arrive(&bar->acc_empty[buf]);
      }
      if (!ok) break;
      // merge: largest key magnitude, smallest column on ties
      uint32_t best_m = 0;
      int best_c = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const uint32_t k = __float_as_uint(acc[i]);
        const uint32_t m = k & 0x7FFFFFF0u;
        const int c = (15 - (int)(k & 15u)) * 32 + i;
        if (m > best_m || (m == best_m && c < best_c)) { best_m = m; best_c = c; }
      }
      // sign of s at the winning column: x . R[:, col] from shared memory
      const int s_idx = it % kStages;
      const uint8_t* xrow = x_smem + s_idx * kXBytes + row_in_tile * 128;
      const uint8_t* rblk = r_smem + (best_c >> 6) * kRBlockBytes;
      const int nn = best_c & 63;
      float dot = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 w = *reinterpret_cast<const uint4*>(xrow + (((uint32_t)c ^ (uint32_t)(row_in_tile & 7)) << 4));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int k = c * 8 + e;
          const float xv = __uint_as_float((e & 1) ? (ws[e >> 1] & 0xffff0000u) : (ws[e >> 1] << 16));
          const uint16_t rb = *reinterpret_cast<const uint16_t*>(
              rblk + k * 128 + ((((uint32_t)nn >> 3) ^ (uint32_t)(k & 7)) << 4) + (nn & 7) * 2);
          dot = fmaf(xv, __uint_as_float((uint32_t)rb << 16), dot);
        }
      }
      mbar_arrive(&bar->x_empty[s_idx]);
      const int64_t row = (int64_t)t * kTileM + row_in_tile;
      if (row < n_rows) {
        const int64_t bh = row / L, pos = row - bh * L;
        bucket[(bh * n_rounds + r) * L + pos] = dot >= 0.f ? best_c : nh + best_c;
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
