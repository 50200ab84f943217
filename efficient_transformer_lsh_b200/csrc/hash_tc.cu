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
// Structure (one CTA per SM, persistent; CTAs are assigned to one round):
//   warp 0  : TMA producer — 128-token X tiles (K-major) through a 4-stage
//             ring, released by the MMAs; R_r as 512-column blocks of the
//             MN-major operand: one block stays resident when n_b/2 <= 512,
//             otherwise the blocks stream through a 2-stage ring, once per
//             pair of X tiles (both tiles use each block);
//   warp 1  : TMEM allocation; one thread issues tcgen05.mma: a 128 x 256 x 64
//             product per 256-column chunk of a block, the chunks of a pair
//             of tiles interleaved;
//   warps 2-5, 6-9: two epilogue warpgroups taking alternate tiles, each with
//             its own 256-column TMEM accumulator (one token per thread).
//             Each s becomes a float key whose 6 low mantissa bits hold
//             (63 - its column / 8 within the block) and whose sign is kept;
//             two 3-input max and min operations fold two columns into each
//             of 8 running maxima (largest +s) and minima (most negative s),
//             one per column mod 8. Keys keep 17 mantissa bits, so values
//             2^-17 (7.6e-6) relative apart still order correctly: equal keys
//             are a near-tie by the 1e-5 bound the results are checked
//             against. After each block the 8 slots are merged into the
//             running best (largest |s|; on ties the +s half, then the lower
//             column).
// Handles n_b/2 a multiple of 8 up to 32768; other shapes use the CUDA-core
// kernel.
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"
#include "tma_host.h"

namespace lsh {
namespace {

using namespace tc;

constexpr int kTileM = 128;          // tokens per tile
constexpr int kStages = 4;           // X ring depth
constexpr int kBlockN = 512;         // rotation columns per R block
constexpr int kChunkN = 256;         // columns per MMA / accumulator
constexpr int kRStages = 2;          // R ring depth when R is streamed
constexpr int kXBytes = kTileM * 128;                    // 16 KB
constexpr int kRBoxBytes = 64 * 128;                     // 64 columns x 64 k-rows
constexpr int kRBlockBytes = (kBlockN / 64) * kRBoxBytes;  // 64 KB
constexpr int kThreads = 320;

struct __align__(8) HashBarriers {
  uint64_t r_full[kRStages];
  uint64_t r_empty[kRStages];
  uint64_t x_full[kStages];
  uint64_t x_empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kSmemBytes =
    1024 + kRStages * kRBlockBytes + kStages * kXBytes + sizeof(HashBarriers);
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

__device__ __forceinline__ bool warp_all(bool ok) { return __all_sync(0xffffffffu, ok); }

// Folds two accumulator values (raw fp32 bits a, b) into the running maximum
// and minimum of one slot, after replacing their 6 low mantissa bits by their
// tags ta, tb (63 - column / 8 within the R block).
__device__ __forceinline__ void fold2(float& mx, float& mn, uint32_t a, uint32_t b, uint32_t ta,
                                      uint32_t tb) {
  const float ka = __uint_as_float((a & 0xFFFFFFC0u) | ta);
  const float kb = __uint_as_float((b & 0xFFFFFFC0u) | tb);
  float r0, r1;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r0) : "f"(mx), "f"(ka), "f"(kb));
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r1) : "f"(mn), "f"(ka), "f"(kb));
  mx = r0;
  mn = r1;
}

// Columns of R block b: [512 b, min(nh, 512 b + 512)).
__device__ __forceinline__ int block_cols(int nh, int b) { return min(kBlockN, nh - b * kBlockN); }

__global__ void __launch_bounds__(kThreads, 1)
hash_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_r,
               int32_t* __restrict__ bucket, int64_t n_rows, int L, int nh, int n_rounds,
               int n_tiles, int ctas_per_round, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* r_smem = smem;
  uint8_t* x_smem = smem + kRStages * kRBlockBytes;
  HashBarriers* bar = (HashBarriers*)(x_smem + kStages * kXBytes);
  volatile int* abort = &bar->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x % n_rounds;
  const int ci = blockIdx.x / n_rounds;
  const int n_blk = (nh + kBlockN - 1) / kBlockN;
  // one R block stays resident; several are streamed through the R ring,
  // once per pair of tiles
  const bool stream_r = n_blk > 1;
  const int n_mine = ci < n_tiles ? (n_tiles - ci + ctas_per_round - 1) / ctas_per_round : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRStages; ++s) {
      mbar_init(&bar->r_full[s], 1);
      mbar_init(&bar->r_empty[s], 1);     // released by the MMAs' commit
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar->x_full[s], 1);
      mbar_init(&bar->x_empty[s], 1);
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
      // R block b into ring stage rs
      auto load_r = [&](int b, int rs) {
        const int nbox = (block_cols(nh, b) + 63) / 64;
        mbar_expect_tx(&bar->r_full[rs], nbox * kRBoxBytes);
        for (int k = 0; k < nbox; ++k)
          tma_load_2d(r_smem + rs * kRBlockBytes + k * kRBoxBytes, &map_r, b * kBlockN + k * 64,
                      r * 64, &bar->r_full[rs]);
      };
      int rb = 0;                            // R blocks loaded
      if (!stream_r) {
        load_r(0, 0);
        rb = 1;
      }
      int it = 0;                            // X tiles loaded
      bool ok = true;
      for (int it0 = 0; it0 < n_mine && ok; it0 += 2) {
        const int cnt = min(2, n_mine - it0);
        for (int k = 0; k < cnt && ok; ++k, ++it) {
          const int s = it % kStages;
          if (it >= kStages &&
              !mbar_wait(&bar->x_empty[s], (uint32_t)(it / kStages - 1) & 1u, abort, status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&bar->x_full[s], kXBytes);
          tma_load_2d(x_smem + s * kXBytes, &map_x, 0, (ci + it * ctas_per_round) * kTileM,
                      &bar->x_full[s]);
        }
        if (stream_r) {
          for (int b = 0; b < n_blk && ok; ++b, ++rb) {
            const int rs = rb % kRStages;
            if (rb >= kRStages &&
                !mbar_wait(&bar->r_empty[rs], (uint32_t)(rb / kRStages - 1) & 1u, abort, status)) {
              ok = false;
              break;
            }
            load_r(b, rs);
          }
        }
      }
      // every issued copy has landed before the CTA may exit (bounded)
      int dummy = 0;
      for (int s = 0; s < kStages && s < it; ++s) {
        const int last = it - 1 - ((it - 1 - s) % kStages);
        mbar_wait(&bar->x_full[s], (uint32_t)(last / kStages) & 1u, (volatile int*)&dummy, status);
      }
      for (int s = 0; s < kRStages && s < rb; ++s) {
        const int last = rb - 1 - ((rb - 1 - s) % kRStages);
        mbar_wait(&bar->r_full[s], (uint32_t)(last / kRStages) & 1u, (volatile int*)&dummy, status);
      }
    }
  } else if (warp == 1) {
    {
      // ---------------- MMA issuer ----------------
      // Tiles alternate between the two accumulators / epilogue warpgroups;
      // the chunks of a pair of tiles are interleaved so both stay busy, and
      // a streamed R block serves both tiles of the pair.
      const uint32_t r_lo = (smem_u32(r_smem) >> 4) | desc_lbo(kRBoxBytes);
      const uint32_t x_lo = (smem_u32(x_smem) >> 4) | desc_lbo(16);
      int uses0 = 0, uses1 = 0, rb = 0;
      bool ok = true;
      if (!stream_r) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bar->r_full[0], 0u, abort, status));
        rb = 1;
      }
      for (int it0 = 0; it0 < n_mine && ok; it0 += 2) {
        const int cnt = min(2, n_mine - it0);
        for (int k = 0; k < cnt && ok; ++k)
          ok = __all_sync(0xffffffffu, mbar_wait(&bar->x_full[(it0 + k) % kStages], (uint32_t)((it0 + k) / kStages) & 1u,
                         abort, status));
        if (!ok) break;
        tc_fence_after();
        for (int b = 0; b < n_blk && ok; ++b) {
          const int rs = stream_r ? rb % kRStages : 0;
          if (stream_r) {
            ok = __all_sync(0xffffffffu, mbar_wait(&bar->r_full[rs], (uint32_t)(rb / kRStages) & 1u, abort, status));
            if (!ok) break;
            tc_fence_after();
          }
          const int bcols = block_cols(nh, b);
          const int nsub = (bcols + kChunkN - 1) / kChunkN;
          for (int j = 0; j < nsub && ok; ++j)
            for (int k = 0; k < cnt && ok; ++k) {
              const int it = it0 + k, w = it & 1, s = it % kStages;
              int& uses = w ? uses1 : uses0;
              if (uses > 0 &&
                  !__all_sync(0xffffffffu, mbar_wait(&bar->acc_empty[w], (uint32_t)(uses - 1) & 1u, abort, status))) {
                ok = false;
                break;
              }
              ++uses;
              tc_fence_after();
              const int ncols = min(kChunkN, bcols - j * kChunkN);
              // whole 64-column boxes: the MN-major operand is read in complete
              // swizzle atoms; the zero-filled extra columns are masked later
              const int n_mma = (ncols + 63) / 64 * 64;
              const uint32_t idesc = idesc_f16(kTileM, n_mma, 1, false, true);
              const uint32_t d = tmem + (uint32_t)(w * kChunkN);
              const uint32_t a = x_lo + (uint32_t)(s * kXBytes) / 16;
              const uint32_t bd =
                  r_lo + (uint32_t)(rs * kRBlockBytes + j * 4 * kRBoxBytes) / 16;
              if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  mma_ss_raw(d, a + 2 * kk, bd + 128 * kk, kDescHi1024, idesc, kk > 0);
                mma_commit_raw(&bar->acc_full[w]);
                if (b == n_blk - 1 && j == nsub - 1) mma_commit_raw(&bar->x_empty[s]);
              }
              __syncwarp();
            }
          if (stream_r && ok) {
            mma_commit(&bar->r_empty[rs]);
            ++rb;
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
    int use = 0;
    bool ok = true;
    for (int it = w; it < n_mine && ok; it += 2) {
      const int t = ci + it * ctas_per_round;
      uint32_t best_m = 0;
      int best_c = 0x7fffffff;
      for (int b = 0; b < n_blk && ok; ++b) {
        // 8 running slots (column mod 8); keys keep 17 mantissa bits, so
        // values 2^-17 (7.6e-6) relative apart still order correctly
        float mx[8], mn[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          mx[k] = -INFINITY;
          mn[k] = INFINITY;
        }
        const int bcols = block_cols(nh, b);
        const int nsub = (bcols + kChunkN - 1) / kChunkN;
        for (int j = 0; j < nsub; ++j, ++use) {
          if (!warp_all(mbar_wait(&bar->acc_full[w], (uint32_t)use & 1u, abort, status))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int ncols = min(kChunkN, bcols - j * kChunkN);
          for (int c0 = 0; c0 < ncols; c0 += 64) {
            uint32_t va[32], vb[32];
            tmem_ld32(tbase + c0, va);
            tmem_ld32(tbase + c0 + 32, vb);     // within the accumulator's 256 columns
            tmem_ld_wait();
            // tag of block column c: 63 - c / 8; va holds 4 column octets,
            // vb the next 4
            const uint32_t t0 = (uint32_t)(63 - (j * kChunkN + c0) / 8);
            if (ncols - c0 >= 64) {
#pragma unroll
              for (int k = 0; k < 8; ++k) {
#pragma unroll
                for (int o = 0; o < 4; o += 2) {
                  fold2(mx[k], mn[k], va[8 * o + k], va[8 * o + 8 + k], t0 - o, t0 - o - 1);
                  fold2(mx[k], mn[k], vb[8 * o + k], vb[8 * o + 8 + k], t0 - 4 - o, t0 - 5 - o);
                }
              }
            } else {
              const int na = ncols - c0, nb = ncols - c0 - 32;
#pragma unroll
              for (int k = 0; k < 8; ++k) {
#pragma unroll
                for (int o = 0; o < 4; o += 2) {
                  // a missing column is a NaN key, which max and min ignore
                  const uint32_t a0 = (8 * o + k < na) ? va[8 * o + k] : 0x7FFFFFFFu;
                  const uint32_t a1 = (8 * o + 8 + k < na) ? va[8 * o + 8 + k] : 0x7FFFFFFFu;
                  const uint32_t b0 = (8 * o + k < nb) ? vb[8 * o + k] : 0x7FFFFFFFu;
                  const uint32_t b1 = (8 * o + 8 + k < nb) ? vb[8 * o + 8 + k] : 0x7FFFFFFFu;
                  fold2(mx[k], mn[k], a0, a1, t0 - o, t0 - o - 1);
                  fold2(mx[k], mn[k], b0, b1, t0 - 4 - o, t0 - 5 - o);
                }
              }
            }
          }
          tc_fence_before();
          mbar_arrive(&bar->acc_empty[w]);
        }
        if (!ok) break;
        // merge the block into the running best: largest |s|; on ties the +s
        // half, then the smaller column
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t kp = __float_as_uint(mx[k]), kn = __float_as_uint(mn[k]);
          // a negative running maximum or a positive running minimum (this
          // includes the initial -inf / +inf) is never the winner
          const bool vp = (kp >> 31) == 0u, vq = (kn >> 31) != 0u;
          const uint32_t mp = vp ? (kp & 0x7FFFFFC0u) : 0u;
          const int cp = vp ? b * kBlockN + (63 - (int)(kp & 63u)) * 8 + k : 0x7fffffff;
          const uint32_t mq = vq ? (kn & 0x7FFFFFC0u) : 0u;
          const int cq = vq ? nh + b * kBlockN + (63 - (int)(kn & 63u)) * 8 + k : 0x7fffffff;
          if (mp > best_m || (mp == best_m && cp < best_c)) { best_m = mp; best_c = cp; }
          if (mq > best_m || (mq == best_m && cq < best_c)) { best_m = mq; best_c = cq; }
        }
      }
      if (!ok) break;
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
  if (p.dtype != LSH_BF16 || nh % 8 != 0 || nh > 32768 || ((uintptr_t)R % 16) != 0)
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
