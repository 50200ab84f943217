// Dense products of the position-wise feed-forward layer that sits beside the
// attention in a Reformer layer ("Reformer: The Efficient Transformer",
// research.elamur.ai summary page, Key points, "Reversible layers": the
// feed-forward layers run chunk by chunk) on the 5th-generation tensor cores:
//
//   C[M x N] = epilogue(A[M x K] B[K x N]),
//
// bf16 operands brought by TMA into 128-byte-swizzled shared memory, fp32
// accumulation in TMEM. Each operand is read either K-major (stored
// [rows][K]) or MN-major (stored [K][rows], i.e. the transpose of a stored
// matrix, as the weight-gradient products need), from a plain row-major
// matrix or from the attention's [B, H, L, 64] activation layout, in which
// token row (b, l) has its 64 H features spread over the H head rows.
//
// Persistent CTAs walk 128 x BN tiles (BN = 64, 128 or 256; K in steps of
// 64) round-robin, with two TMEM accumulators so that one tile's epilogue
// runs under the next tile's products. The operand loads are latency-bound
// (L2 and the TMA read path run well below their peaks), so what sets the
// rate is the bytes in flight per SM: two CTAs with 3-stage rings for
// BN <= 128, one CTA with a 4-stage ring for BN = 256.
//   warp 0     : one lane issues the TMA loads into the ring;
//   warp 1     : TMEM allocation; one lane issues the MMAs (128 x BN x 16);
//   warps 2-9  : epilogue, two warpgroups each taking half of the columns,
//                one thread per tile row (TMEM lane): bias, ReLU, mask,
//                residual, then bf16 or fp32 stores (optionally
//                accumulating into fp32), releasing the accumulator as soon
//                as it is read.
// Every output element's K sum runs in the same order whichever tile or
// launch computes its row, so splitting the rows into chunks does not change
// a single bit of the result.
#include <cuda_bf16.h>
#include <stddef.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"
#include "tma_host.h"

namespace lsh {
namespace {

using namespace tc;

constexpr int kBM = 128, kBK = 64;
constexpr int kThreads = 320;
constexpr int kATile = kBM * kBK * 2;   // 16 KB
constexpr int kMaxSplits = kGemmMaxSplits;

// Ring depth and CTAs per SM by tile width: two CTAs with 3 stages each for
// BN <= 128 (2 x 2 x BN TMEM columns), one CTA with 4 stages for BN = 256
// (its two accumulators take all 512 TMEM columns).
template <int BN>
struct GemmCfg {
  static constexpr int kStages = BN == 256 ? 4 : 3;
  static constexpr int kCtasPerSm = BN == 256 ? 1 : 2;
};

template <int kStages>
struct __align__(8) GemmBar {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_base;
  int abort;
};

template <int BN>
constexpr size_t gemm_smem() {
  constexpr int S = GemmCfg<BN>::kStages;
  return 1024 + (size_t)S * (kATile + BN * kBK * 2) + sizeof(GemmBar<S>);
}

// Coordinates of the box whose first row is `row` (along the map's row
// dimension) and whose 64 inner elements are block `blk` of the inner
// dimension: plain maps are (cols, rows, 1, 1); head-layout maps are
// (64, L, H, B) with token row r = b L + l and head h = blk.
__device__ __forceinline__ void load_box(void* dst, const CUtensorMap* map, int heads, int L,
                                         int64_t row, int blk, uint64_t* bar) {
  if (heads)
    tma_load_4d(dst, map, 0, (int32_t)(row % L), blk, (int32_t)(row / L), bar);
  else
    tma_load_4d(dst, map, blk * 64, (int32_t)row, 0, 0, bar);
}

// Eight floats (v[o .. o + 7]) to a 32-byte aligned address in one store.
__device__ __forceinline__ void st_v8(float* p, const float (&v)[16], int o) {
  asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "f"(v[o]),
               "f"(v[o + 1]), "f"(v[o + 2]), "f"(v[o + 3]), "f"(v[o + 4]), "f"(v[o + 5]),
               "f"(v[o + 6]), "f"(v[o + 7])
               : "memory");
}

// Tile t of the product: M tile fastest, then N tile, then K split.
struct TileCoord {
  int m0, n0, z;
};
__device__ __forceinline__ TileCoord tile_coord(int t, int tiles_m, int tiles_n, int bn) {
  TileCoord c;
  c.m0 = (t % tiles_m) * kBM;
  t /= tiles_m;
  c.n0 = (t % tiles_n) * bn;
  c.z = t / tiles_n;
  return c;
}

template <int BN>
__global__ void __launch_bounds__(kThreads, GemmCfg<BN>::kCtasPerSm)
gemm_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
               GemmOpDev a, GemmOpDev b, int K, GemmEpi e, int tiles_m, int tiles_n, int splits,
               int wide, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sa = smem;
  constexpr int kStages = GemmCfg<BN>::kStages;
  uint8_t* sb = smem + kStages * kATile;
  constexpr int kBTile = BN * kBK * 2;
  GemmBar<kStages>* bar = (GemmBar<kStages>*)(sb + kStages * kBTile);
  volatile int* abort = &bar->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = tiles_m * tiles_n * splits;
  const int nk = K / kBK / splits;   // K blocks per split

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar->full[s], 1);
      mbar_init(&bar->empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bar->acc_full[x], 1);
      mbar_init(&bar->acc_empty[x], 256);
    }
    bar->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar->tmem_base, 2 * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp == 0) {
    // ---------------------------------------------- TMA producer
    if (elect_one()) {
      prefetch_tmap(&map_a);
      prefetch_tmap(&map_b);
      int q = 0;   // ring slots used so far
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        const TileCoord tc = tile_coord(t, tiles_m, tiles_n, BN);
        const int kb0 = tc.z * nk;
        for (int kb = 0; kb < nk; ++kb, ++q) {
          const int s = q % kStages;
          if (q >= kStages &&
              !mbar_wait(&bar->empty[s], (uint32_t)(q / kStages - 1) & 1u, abort, status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&bar->full[s], (uint32_t)(kATile + kBTile));
          uint8_t* da = sa + s * kATile;
          uint8_t* db = sb + s * kBTile;
          if (a.mn_major) {
            load_box(da, &map_a, a.heads, a.L, a.row0 + (int64_t)(kb0 + kb) * kBK, tc.m0 / 64,
                     &bar->full[s]);
            load_box(da + kATile / 2, &map_a, a.heads, a.L, a.row0 + (int64_t)(kb0 + kb) * kBK,
                     tc.m0 / 64 + 1, &bar->full[s]);
          } else {
            load_box(da, &map_a, a.heads, a.L, a.row0 + tc.m0, kb0 + kb, &bar->full[s]);
          }
          if (b.mn_major) {
#pragma unroll
            for (int i = 0; i < BN / 64; ++i)
              load_box(db + i * (64 * 128), &map_b, b.heads, b.L,
                       b.row0 + (int64_t)(kb0 + kb) * kBK, tc.n0 / 64 + i, &bar->full[s]);
          } else {
            load_box(db, &map_b, b.heads, b.L, b.row0 + tc.n0, kb0 + kb, &bar->full[s]);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------- MMA issuer: tiles alternate
    // between the two accumulators, so one tile's epilogue overlaps the next
    // tile's products
    constexpr uint32_t kLboMN = desc_lbo(64 * 128);   // 64-wide M/N blocks, 8 KB apart
    const uint32_t idesc = idesc_f16(kBM, BN, 1, a.mn_major != 0, b.mn_major != 0);
    const uint32_t a_lbo = a.mn_major ? kLboMN : desc_lbo(16);
    const uint32_t b_lbo = b.mn_major ? kLboMN : desc_lbo(16);
    const uint32_t a_step = a.mn_major ? 128u : 2u;   // one K step of 16, in 16-byte units
    const uint32_t b_step = b.mn_major ? 128u : 2u;
    bool ok = true;
    int q = 0, i = 0;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++i) {
      const int x = i & 1;
      if (i >= 2)
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&bar->acc_empty[x], (uint32_t)(i / 2 - 1) & 1u, abort, status));
      if (!ok) break;
      tc_fence_after();
      const uint32_t d = tmem + (uint32_t)(x * BN);
      for (int kb = 0; kb < nk && ok; ++kb, ++q) {
        const int s = q % kStages;
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&bar->full[s], (uint32_t)(q / kStages) & 1u, abort, status));
        if (!ok) break;
        tc_fence_after();
        const uint32_t alo = (smem_u32(sa + s * kATile) >> 4) | a_lbo;
        const uint32_t blo = (smem_u32(sb + s * kBTile) >> 4) | b_lbo;
        if (elect_one()) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_ss_raw(d, alo + a_step * ks, blo + b_step * ks, kDescHi1024, idesc,
                       (kb > 0 || ks > 0) ? 1u : 0u);
          mma_commit_raw(&bar->empty[s]);
        }
        __syncwarp();
      }
      mma_commit(&bar->acc_full[x]);
    }
  } else {
    // ---------------------------------------------- epilogue
    const int qw = warp & 3;             // TMEM lane quarter of this warp
    const int cb = ((warp - 2) >> 2) * (BN / 2);   // this warpgroup's column half
    const int r = qw * 32 + lane;        // tile row
    int i = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      const int x = i & 1;
      const TileCoord tc = tile_coord(t, tiles_m, tiles_n, BN);
      const bool got =
          __all_sync(0xffffffffu, mbar_wait(&bar->acc_full[x], (uint32_t)(i / 2) & 1u, abort, status));
      if (!got) break;
      tc_fence_after();
      const int64_t row = (int64_t)tc.m0 + r;
      const bool live = row < e.M;
      const int64_t orow = e.row0 + row;
      // element offset of (orow, column c) in the output / residual layout
      auto out_off = [&](int c) -> int64_t {
        if (e.out_heads) {
          const int64_t bb = orow / e.L, l = orow - bb * e.L;
          return ((bb * e.H + c / 64) * e.L + l) * 64 + (c & 63);
        }
        return orow * e.ldo + c;
      };
#pragma unroll 1
      for (int c0 = cb; c0 < cb + BN / 2; c0 += 16) {
        uint32_t acc[16];
        tmem_ld16(tmem + ((uint32_t)(qw * 32) << 16) + (uint32_t)(x * BN + c0), acc);
        tmem_ld_wait();
        if (c0 + 16 >= cb + BN / 2) {
          // every TMEM read of this accumulator is done: release it to the MMAs
          tc_fence_before();
          mbar_arrive(&bar->acc_empty[x]);
        }
        if (!live) continue;
        const int c = tc.n0 + c0;
        float v[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) v[k] = __uint_as_float(acc[k]);
        if (e.split_part) {
          // one K split's raw sums; split_reduce_kernel adds the splits
          float* sp = e.split_part + ((int64_t)tc.z * e.M + row) * e.ldo + c;
          if (wide) {
            st_v8(sp, v, 0);
            st_v8(sp + 8, v, 8);
          } else {
            float4* op = reinterpret_cast<float4*>(sp);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              op[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
          }
          continue;
        }
        if (e.bias) {
#pragma unroll
          for (int k = 0; k < 16; ++k) v[k] += __ldg(e.bias + c + k);
        }
        if (e.relu) {
#pragma unroll
          for (int k = 0; k < 16; ++k) v[k] = fmaxf(v[k], 0.f);
        }
        if (e.mask) {
          const uint4* mp = reinterpret_cast<const uint4*>(e.mask + row * e.ldm + c);
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const uint4 w = __ldg(mp + k);
            const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              if (!(__uint_as_float(u[m] << 16) > 0.f)) v[8 * k + 2 * m] = 0.f;
              if (!(__uint_as_float(u[m] & 0xffff0000u) > 0.f)) v[8 * k + 2 * m + 1] = 0.f;
            }
          }
        }
        const int64_t off = out_off(c);
        if (e.res) {
          const uint4* rp = reinterpret_cast<const uint4*>(e.res + off);
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const uint4 w = __ldg(rp + k);
            const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              v[8 * k + 2 * m] = fmaf(e.res_sign, v[8 * k + 2 * m], __uint_as_float(u[m] << 16));
              v[8 * k + 2 * m + 1] =
                  fmaf(e.res_sign, v[8 * k + 2 * m + 1], __uint_as_float(u[m] & 0xffff0000u));
            }
          }
        }
        if (e.out_f32) {
          float4* op = reinterpret_cast<float4*>((float*)e.out + off);
          if (e.accumulate) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float4 pp = op[k];
              v[4 * k] += pp.x;
              v[4 * k + 1] += pp.y;
              v[4 * k + 2] += pp.z;
              v[4 * k + 3] += pp.w;
            }
          }
          if (wide) {
            st_v8((float*)e.out + off, v, 0);
            st_v8((float*)e.out + off + 8, v, 8);
          } else {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              op[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
          }
        } else {
          uint32_t pk[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
            pk[k] = *reinterpret_cast<uint32_t*>(&h2);
          }
          if (wide) {
            asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(
                             (__nv_bfloat16*)e.out + off),
                         "r"(pk[0]), "r"(pk[1]), "r"(pk[2]), "r"(pk[3]), "r"(pk[4]), "r"(pk[5]),
                         "r"(pk[6]), "r"(pk[7])
                         : "memory");
          } else {
            uint4* op = reinterpret_cast<uint4*>((__nv_bfloat16*)e.out + off);
            op[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            op[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * BN);
  }
}

// out (+)= the S splits' partial sums, added in split order (float4 units).
__global__ void __launch_bounds__(256)
split_reduce_kernel(const float* __restrict__ part, int S, int64_t n4, float* __restrict__ out,
                    int accumulate) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  float4 a = accumulate ? reinterpret_cast<const float4*>(out)[i] : make_float4(0.f, 0.f, 0.f, 0.f);
  for (int z = 0; z < S; ++z) {
    const float4 p = __ldg(reinterpret_cast<const float4*>(part) + z * n4 + i);
    a.x += p.x;
    a.y += p.y;
    a.z += p.z;
    a.w += p.w;
  }
  reinterpret_cast<float4*>(out)[i] = a;
}

// Tensor map of one operand: plain (cols, rows, 1, 1) or head layout
// (64, L, H, B); box of 64 inner elements by `box_rows` rows.
bool encode_op(CUtensorMap* map, const GemmOpHost& o, uint32_t box_rows) {
  uint64_t dims[4], strides[3];
  const uint32_t box[4] = {64, box_rows, 1, 1};
  if (o.heads) {
    dims[0] = 64;
    dims[1] = (uint64_t)o.L;
    dims[2] = (uint64_t)o.H;
    dims[3] = (uint64_t)o.B;
    strides[0] = 128;
    strides[1] = (uint64_t)o.L * 128;
    strides[2] = (uint64_t)o.H * o.L * 128;
  } else {
    dims[0] = (uint64_t)o.cols;
    dims[1] = (uint64_t)o.rows;
    dims[2] = 1;
    dims[3] = 1;
    strides[0] = (uint64_t)o.cols * 2;
    strides[1] = strides[0] * (uint64_t)o.rows;
    strides[2] = strides[1];
  }
  return encode_tmap_4d_16bit(map, o.base, dims, strides, box);
}

template <int BN>
cudaError_t launch_bn(const GemmOpHost& a, const GemmOpHost& b, int M, int N, int K, int splits,
                      const GemmEpi& e, int* status, cudaStream_t s) {
  CUtensorMap ma, mb;
  if (!encode_op(&ma, a, a.mn_major ? 64 : kBM) || !encode_op(&mb, b, b.mn_major ? 64 : BN))
    return cudaErrorInvalidValue;
  const GemmOpDev da{a.mn_major, a.heads, a.L, a.row0};
  const GemmOpDev db{b.mn_major, b.heads, b.L, b.row0};
  constexpr size_t smem = gemm_smem<BN>();
  cudaError_t err =
      cudaFuncSetAttribute(gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int tiles_m = (M + kBM - 1) / kBM, tiles_n = N / BN;
  const int n_tiles = tiles_m * tiles_n * splits;
  const int grid = std::min(n_tiles, GemmCfg<BN>::kCtasPerSm * sm_count());
  // 256-bit stores when every 16-column piece of a row starts on 32 bytes:
  // the base pointers 32-byte aligned and plain rows a multiple of 16
  // elements apart (head-layout rows are 64 elements)
  const bool wide = ((uintptr_t)e.out & 31) == 0 && ((uintptr_t)e.split_part & 31) == 0 &&
                    (e.out_heads || e.ldo % 16 == 0);
  gemm_tc_kernel<BN><<<grid, kThreads, smem, s>>>(ma, mb, da, db, K, e, tiles_m, tiles_n, splits,
                                                   wide ? 1 : 0, status);
  note_launch();
  if (e.split_part) {
    const int64_t n4 = (int64_t)M * N / 4;
    split_reduce_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, s>>>(
        e.split_part, splits, n4, (float*)e.out, e.accumulate);
    note_launch();
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_tc(const GemmOpHost& a, const GemmOpHost& b, int M, int N, int K,
                           const GemmEpi& e, int* status, cudaStream_t s) {
  if (M <= 0 || N <= 0 || K <= 0 || K % kBK != 0 || N % 64 != 0) return cudaErrorInvalidValue;
  // the K-split (weight-gradient) products have long K and few tiles: the
  // 256-wide tile moves a third fewer operand bytes per MMA; the others run
  // faster as two 128-wide CTAs per SM
  const int bn = (e.split_part && N % 256 == 0) ? 256 : N % 128 == 0 ? 128 : 64;
  int splits = 1;
  if (e.split_part) {
    // a plain float32 product (no epilogue terms) with few tiles: split K
    // so that about one CTA per SM runs, in pieces of at least 4 K blocks
    if (!e.out_f32 || e.out_heads || e.bias || e.relu || e.mask || e.res || e.ldo != N ||
        e.row0 != 0)
      return cudaErrorInvalidValue;
    const int tiles = ((M + kBM - 1) / kBM) * (N / bn);
    const int nk = K / kBK;
    while (splits < kMaxSplits && tiles * splits * 2 <= sm_count() && nk % (splits * 2) == 0 &&
           nk / (splits * 2) >= 4)
      splits *= 2;
  }
  GemmEpi e2 = e;
  if (splits == 1) e2.split_part = nullptr;
  if (bn == 256) return launch_bn<256>(a, b, M, N, K, splits, e2, status, s);
  if (bn == 128) return launch_bn<128>(a, b, M, N, K, splits, e2, status, s);
  return launch_bn<64>(a, b, M, N, K, splits, e2, status, s);
}

}  // namespace lsh
