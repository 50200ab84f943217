// Stable sort of positions by bucket, one segment per (batch, head, round).
//
// "Reformer: The Efficient Transformer" (research.elamur.ai summary page),
// Summary and Key points "LSH attention": positions are sorted by bucket
// before chunking. Sorting stably by bucket is sorting by the packed key
// (round, bucket, position), because positions arrive in increasing order.
//
// Counting sort. Two paths:
//  * n_buckets <= 8192 (every shape the workloads use): two kernels over
//    blocks of 8K-32K consecutive positions, one CTA each (see the counting
//    path below): block totals per bucket from shared-memory atomics, then a
//    scatter kernel that ranks positions within each warp step by a warp
//    bitonic sort of (bucket, lane) keys; the bucket bases come from the
//    scatter kernel itself, or, for many blocks or few segments, from two
//    small scan kernels;
//  * larger bucket counts: per 4096-position tile the packed keys
//    (bucket << 12 | local index) are sorted in shared memory by a bitonic
//    network; row_scan / bucket_scan form the bases; scatter places them.
// Ranks follow position order inside a warp step (the lane breaks ties),
// across the steps of a warp (in order), across the warps of a block
// (exclusive prefix of their counts) and across blocks (counts of the blocks
// before), so the whole sort is stable.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace lsh {
namespace {

constexpr int kTile = 4096;        // positions per tile (12-bit local index)
constexpr int kTileThreads = 1024;

__device__ __forceinline__ void bitonic_sort_smem(uint32_t* s) {
  const int tid = threadIdx.x;
  for (int k = 2; k <= kTile; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int e = tid; e < kTile / 2; e += kTileThreads) {
        int i = (e / j) * 2 * j + (e % j);
        int ip = i + j;
        bool up = (i & k) == 0;
        uint32_t a = s[i], b = s[ip];
        if ((a > b) == up) { s[i] = b; s[ip] = a; }
      }
      __syncthreads();
    }
  }
}

// First index in the sorted tile whose bucket is >= b.
__device__ __forceinline__ int lower_bound_bucket(const uint32_t* s, uint32_t b) {
  uint32_t key = b << 12;
  int lo = 0, hi = kTile;
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (s[mid] < key) lo = mid + 1; else hi = mid;
  }
  return lo;
}

__global__ void __launch_bounds__(kTileThreads)
tile_sort_kernel(const int32_t* __restrict__ bucket, uint32_t* __restrict__ sorted,
                 int32_t* __restrict__ counts, int L, int n_buckets, int tiles, int* status) {
  __shared__ uint32_t s[kTile];
  const int tile = blockIdx.x % tiles;
  const int64_t seg = blockIdx.x / tiles;
  const int64_t p0 = (int64_t)tile * kTile;
  const int n = min(kTile, (int)(L - p0));
  const int32_t* src = bucket + seg * L + p0;
  for (int i = threadIdx.x; i < kTile; i += kTileThreads) {
    uint32_t key = 0xffffffffu;
    if (i < n) {
      uint32_t b = (uint32_t)src[i];
      if (b >= (uint32_t)n_buckets) {   // out-of-range id: flag it, keep memory safe
        record_status(status, (int)LSH_ERR_DEVICE_CHECK);
        b = (uint32_t)n_buckets - 1;
      }
      key = (b << 12) | (uint32_t)i;
    }
    s[i] = key;
  }
  __syncthreads();
  bitonic_sort_smem(s);
  uint32_t* dst = sorted + seg * L + p0;
  for (int i = threadIdx.x; i < n; i += kTileThreads) {
    uint32_t key = s[i];
    dst[i] = key;
    uint32_t b = key >> 12;
    bool last = (i == n - 1) || ((s[i + 1] >> 12) != b);
    if (last) {
      int first = lower_bound_bucket(s, b);
      counts[(seg * n_buckets + b) * tiles + tile] = i - first + 1;
    }
  }
}

// One warp per (seg, bucket): exclusive scan of counts over tiles; writes the
// bucket total to base[seg][bucket].
__global__ void row_scan_kernel(int32_t* __restrict__ counts, int32_t* __restrict__ base,
                                int64_t rows, int tiles) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  int32_t* c = counts + row * tiles;
  int carry = 0;
  for (int t0 = 0; t0 < tiles; t0 += 32) {
    int t = t0 + lane;
    int v = (t < tiles) ? c[t] : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (t < tiles) c[t] = carry + x - v;
    carry += __shfl_sync(0xffffffffu, x, 31);
  }
  if (lane == 0) base[row] = carry;
}

// One block per segment: exclusive scan of the bucket totals, in place.
__global__ void __launch_bounds__(1024)
bucket_scan_kernel(int32_t* __restrict__ base, int n_buckets) {
  __shared__ int warp_tot[32];
  __shared__ int carry_s;
  int32_t* b = base + (int64_t)blockIdx.x * n_buckets;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry_s = 0;
  __syncthreads();
  for (int i0 = 0; i0 < n_buckets; i0 += 1024) {
    int i = i0 + threadIdx.x;
    int v = (i < n_buckets) ? b[i] : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = warp_tot[lane];
      int wx = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, wx, o);
        if (lane >= o) wx += y;
      }
      warp_tot[lane] = wx - w;   // exclusive prefix of warp totals
    }
    __syncthreads();
    int carry = carry_s;
    if (i < n_buckets) b[i] = carry + warp_tot[warp] + x - v;
    __syncthreads();
    if (threadIdx.x == 1023) carry_s = carry + warp_tot[31] + x;
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kTileThreads)
scatter_kernel(const uint32_t* __restrict__ sorted, const int32_t* __restrict__ counts,
               const int32_t* __restrict__ base, int32_t* __restrict__ perm, int L,
               int n_buckets, int tiles) {
  __shared__ uint32_t s[kTile];
  const int tile = blockIdx.x % tiles;
  const int64_t seg = blockIdx.x / tiles;
  const int64_t p0 = (int64_t)tile * kTile;
  const int n = min(kTile, (int)(L - p0));
  const uint32_t* src = sorted + seg * L + p0;
  for (int i = threadIdx.x; i < kTile; i += kTileThreads) s[i] = (i < n) ? src[i] : 0xffffffffu;
  __syncthreads();
  int32_t* out = perm + seg * L;
  for (int i = threadIdx.x; i < n; i += kTileThreads) {
    uint32_t key = s[i];
    uint32_t b = key >> 12;
    int first = lower_bound_bucket(s, b);
    int64_t row = seg * n_buckets + b;
    int slot = base[row] + counts[row * tiles + tile] + (i - first);
    out[slot] = (int32_t)(p0 + (key & 0xfffu));
  }
}

// ---- counting path (n_buckets <= kWarpMaxBuckets) -------------------------
// A segment is cut into Q blocks of P consecutive positions, one CTA each;
// warp w of a CTA owns PW consecutive positions of its block.
//   sort_count_kernel:   counts[seg][q][bucket] = the block's bucket totals,
//                        from shared-memory atomics (every bucket written, so
//                        no clearing pass is needed);
//   sort_scatter_kernel: bucket bases of the segment (exclusive scan of the
//                        totals over buckets) plus the counts of the blocks
//                        before q; then each warp takes its positions 32 at a
//                        time, sorts the 32 (bucket, lane) keys with a warp
//                        bitonic network so equal buckets form contiguous
//                        segments in lane order, and ranks each position
//                        within its segment. A first pass counts per warp, an
//                        exclusive prefix over warps gives each warp's run, and
//                        a second pass places every position at its slot.
//   sort_qscan_kernel,
//   sort_bscan_kernel:   (when Q * n_buckets is large or S * Q small) the
//                        prefix over blocks and the bucket bases, so that the
//                        scatter kernel reads two numbers per bucket.
constexpr int kWarpMaxBuckets = 8192;
constexpr int kSortSmemBudget = 200 * 1024;

struct WarpGeo {
  int W;        // warps per CTA
  int PW;       // positions per warp (multiple of 32)
  int P;        // positions per CTA = W * PW
  int Q;        // CTAs per segment
  bool scanned; // block prefixes and bucket bases from the two scan kernels
  size_t smem;  // dynamic shared memory of the scatter kernel (the larger)
};

constexpr int64_t kDirectCounts = 65536;   // Q * n_buckets read by each scatter CTA at most

WarpGeo warp_geo(const lsh_problem& p) {
  WarpGeo g;
  const int nb = p.n_buckets;
  const int64_t S = (int64_t)p.B * p.H * p.n_rounds;
  g.W = (int)std::min<int64_t>(32, (kSortSmemBudget - 8 * (int64_t)nb) / (2 * (int64_t)nb));
  // a few blocks per segment (at most ~16) of 8K..32K positions
  int64_t P = std::min<int64_t>(32768, std::max<int64_t>(8192, ((int64_t)p.L + 15) / 16));
  int64_t Q = ((int64_t)p.L + P - 1) / P;
  if (S * Q > 2 * 148 && p.L <= 32768) {
    // more CTAs than one wave of two per SM: one block per segment instead
    // (no ragged second block)
    P = p.L;
    Q = 1;
  }
  g.scanned = Q * nb > kDirectCounts || S * Q < 148;
  if (g.scanned) {
    // smaller blocks, about one CTA per SM over all segments (each CTA's
    // fixed work grows with W x n_buckets, so fewer, longer CTAs pay when
    // n_buckets is large); the scan kernels then give each CTA its bases
    P = std::min<int64_t>(32768, std::max<int64_t>(32 * g.W, S * p.L / 148));
  }
  g.PW = (int)((P + 32 * g.W - 1) / (32 * g.W)) * 32;
  g.P = g.W * g.PW;
  g.Q = (int)(((int64_t)p.L + g.P - 1) / g.P);
  // per-warp counters, bucket bases, block prefixes (not on the scanned
  // path, whose bases already include them) and 64 words of scratch
  g.smem = (size_t)g.W * nb * 2 + (size_t)nb * (g.scanned ? 4 : 8) + 64 * 4;
  return g;
}

// Bucket of position i of the segment (0xffffffff past the end); an id
// outside [0, n_buckets) is recorded and replaced by n_buckets - 1.
__device__ __forceinline__ uint32_t load_bucket(const int32_t* __restrict__ seg_bucket, int64_t i,
                                                int L, int n_buckets, int* status) {
  if (i >= L) return 0xffffffffu;
  uint32_t b = (uint32_t)__ldg(seg_bucket + i);
  if (b >= (uint32_t)n_buckets) {
    record_status(status, (int)LSH_ERR_DEVICE_CHECK);
    b = (uint32_t)n_buckets - 1;
  }
  return b;
}

// Sorts the warp's 32 keys ascending (bitonic network over lanes).
__device__ __forceinline__ uint32_t warp_sort32(uint32_t key, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const uint32_t o = __shfl_xor_sync(0xffffffffu, key, j);
      const bool up = (lane & k) == 0, lower = (lane & j) == 0;
      key = (lower == up) ? min(key, o) : max(key, o);
    }
  }
  return key;
}

// One step of 32 positions: after sorting (bucket << 5 | lane) keys, lane k
// holds sorted entry k: its bucket, the lane (position offset) it came from,
// its rank among the entries of its bucket, and whether it ends the bucket's
// segment (then `len` is the segment's length).
struct StepRank {
  uint32_t bucket;
  int src, rank, len;
  bool live, last;
};
__device__ __forceinline__ StepRank rank_sorted(uint32_t key, int lane) {
  StepRank r;
  r.live = key != 0xffffffffu;
  r.bucket = key >> 5;
  r.src = (int)(key & 31u);
  const uint32_t prev = __shfl_up_sync(0xffffffffu, r.bucket, 1);
  const uint32_t next = __shfl_down_sync(0xffffffffu, r.bucket, 1);
  const bool first = lane == 0 || prev != r.bucket;
  r.last = lane == 31 || next != r.bucket;
  const uint32_t starts = __ballot_sync(0xffffffffu, first);
  const int seg0 = 31 - __clz(starts & (0xffffffffu >> (31 - lane)));
  r.rank = lane - seg0;
  r.len = r.rank + 1;
  return r;
}
__device__ __forceinline__ uint32_t step_key(uint32_t b, int lane) {
  return warp_sort32(b == 0xffffffffu ? 0xffffffffu : (b << 5) | (uint32_t)lane, lane);
}
__device__ __forceinline__ StepRank rank_step(uint32_t b, int lane) {
  return rank_sorted(step_key(b, lane), lane);
}

__global__ void __launch_bounds__(1024)
sort_count_kernel(const int32_t* __restrict__ bucket, int32_t* __restrict__ counts, int L,
                  int n_buckets, int P, int Q, int* status) {
  extern __shared__ __align__(16) uint8_t sm[];
  uint32_t* cnt = reinterpret_cast<uint32_t*>(sm);      // [n_buckets]
  const int q = blockIdx.x % Q;
  const int64_t seg = blockIdx.x / Q;
  for (int b = threadIdx.x; b < n_buckets; b += blockDim.x) cnt[b] = 0u;
  __syncthreads();
  const int32_t* sb = bucket + seg * L;
  const int64_t p0 = (int64_t)q * P;
  for (int i = threadIdx.x; i < P; i += blockDim.x) {
    const uint32_t b = load_bucket(sb, p0 + i, L, n_buckets, status);
    if (b != 0xffffffffu) atomicAdd(&cnt[b], 1u);
  }
  __syncthreads();
  int32_t* out = counts + (seg * Q + q) * (int64_t)n_buckets;
  for (int b = threadIdx.x; b < n_buckets; b += blockDim.x) out[b] = (int32_t)cnt[b];
}

// Exclusive scan of v[0, n) in place by the whole block; `red` holds 64 ints
// of scratch.
__device__ __forceinline__ void block_exclusive_scan(int32_t* v, int n, int* red) {
  const int T = blockDim.x, t = threadIdx.x, lane = t & 31, w = t >> 5;
  const int per = (n + T - 1) / T;
  const int lo = min(n, t * per), hi = min(n, lo + per);
  int sum = 0;
  for (int i = lo; i < hi; ++i) sum += v[i];
  int x = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) red[w] = x;
  __syncthreads();
  if (w == 0) {
    const int nw = (T + 31) >> 5;
    const int a = lane < nw ? red[lane] : 0;
    int y = a;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int z = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) y += z;
    }
    red[32 + lane] = y - a;   // exclusive prefix of the warp sums
  }
  __syncthreads();
  int run = red[32 + w] + x - sum;
  for (int i = lo; i < hi; ++i) {
    const int c = v[i];
    v[i] = run;
    run += c;
  }
  __syncthreads();
}

// For every (segment, bucket): exclusive prefix of the block counts over the
// blocks, in place, and the bucket's total.
__global__ void __launch_bounds__(256)
sort_qscan_kernel(int32_t* __restrict__ counts, int32_t* __restrict__ totals, int n_buckets, int Q,
                  int64_t rows) {
  const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;   // seg * n_buckets + b
  if (k >= rows) return;
  const int64_t seg = k / n_buckets, b = k - seg * n_buckets;
  int32_t* c = counts + seg * Q * (int64_t)n_buckets + b;
  int run = 0;
  // eight blocks' counts loaded before any is replaced, so their latencies
  // overlap
  for (int q0 = 0; q0 < Q; q0 += 8) {
    int v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = q0 + u < Q ? c[(int64_t)(q0 + u) * n_buckets] : 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (q0 + u < Q) c[(int64_t)(q0 + u) * n_buckets] = run;
      run += v[u];
    }
  }
  totals[k] = run;
}

// For every segment: exclusive scan of the bucket totals, in place (the
// bucket bases).
__global__ void __launch_bounds__(1024)
sort_bscan_kernel(int32_t* __restrict__ totals, int n_buckets) {
  __shared__ int red[64];
  block_exclusive_scan(totals + (int64_t)blockIdx.x * n_buckets, n_buckets, red);
}

// kCache: pass 1 keeps each step's sorted keys in shared memory (4 bytes a
// position, after the counters), so pass 2 only ranks them again.
template <bool kCache>
__global__ void __launch_bounds__(1024)
sort_scatter_kernel(const int32_t* __restrict__ bucket, const int32_t* __restrict__ counts,
                    const int32_t* __restrict__ bases, int32_t* __restrict__ perm, int L,
                    int n_buckets, int PW, int P, int Q) {
  extern __shared__ __align__(16) uint8_t sm[];
  const int W = blockDim.x >> 5;
  uint16_t* cnt = reinterpret_cast<uint16_t*>(sm);                                // [W][nb]
  int32_t* base = reinterpret_cast<int32_t*>(sm + (size_t)W * n_buckets * 2);     // [nb]
  int32_t* pre = base + n_buckets;                                                 // [nb], unless scanned
  int* red = pre + (bases ? 0 : n_buckets);                                        // [64]
  uint32_t* keys = reinterpret_cast<uint32_t*>(red + 64);                          // [W][PW]
  const int q = blockIdx.x % Q;
  const int64_t seg = blockIdx.x / Q;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  {
    uint32_t* c32 = reinterpret_cast<uint32_t*>(cnt);   // W * n_buckets is even
    for (int i = threadIdx.x; i < W * n_buckets / 2; i += blockDim.x) c32[i] = 0u;
  }
  const int32_t* cs = counts + seg * Q * (int64_t)n_buckets;
  if (bases) {
    // from the scan kernels: bucket bases, and the counts before this block
    const int32_t* bs = bases + seg * (int64_t)n_buckets;
    for (int b = threadIdx.x; b < n_buckets; b += blockDim.x)
      base[b] = __ldg(bs + b) + __ldg(cs + (int64_t)q * n_buckets + b);
    __syncthreads();
  } else {
    // totals of the segment per bucket, and the counts of the blocks before q
    for (int b = threadIdx.x; b < n_buckets; b += blockDim.x) {
      int tot = 0, before = 0;
      for (int qq = 0; qq < Q; ++qq) {
        const int c = __ldg(cs + (int64_t)qq * n_buckets + b);
        tot += c;
        if (qq < q) before += c;
      }
      base[b] = tot;
      pre[b] = before;
    }
    __syncthreads();
    block_exclusive_scan(base, n_buckets, red);
    for (int b = threadIdx.x; b < n_buckets; b += blockDim.x) base[b] += pre[b];
  }
  const int32_t* sbk = bucket + seg * L;
  const int64_t i0 = (int64_t)q * P + (int64_t)w * PW;
  uint16_t* mine = cnt + w * n_buckets;
  // pass 1: this warp's count of every bucket
  for (int st = 0; st < PW; st += 32) {
    const uint32_t b = load_bucket(sbk, i0 + st + lane, L, n_buckets, nullptr);
    const uint32_t key = step_key(b, lane);
    if (kCache) keys[w * PW + st + lane] = key;
    const StepRank r = rank_sorted(key, lane);
    if (r.live && r.last) mine[r.bucket] = (uint16_t)(mine[r.bucket] + r.len);
    __syncwarp();
  }
  __syncthreads();
  // exclusive prefix over warps: cnt[w][b] becomes the start of warp w's run
  for (int b = threadIdx.x; b < n_buckets; b += blockDim.x) {
    int acc = 0;
    for (int ww = 0; ww < W; ++ww) {
      const int c = cnt[ww * n_buckets + b];
      cnt[ww * n_buckets + b] = (uint16_t)acc;
      acc += c;
    }
  }
  __syncthreads();
  // pass 2: every position to base + warp run + earlier steps + rank
  int32_t* out = perm + seg * L;
  for (int st = 0; st < PW; st += 32) {
    StepRank r;
    if (kCache) {
      r = rank_sorted(keys[w * PW + st + lane], lane);
    } else {
      const uint32_t b = load_bucket(sbk, i0 + st + lane, L, n_buckets, nullptr);
      r = rank_step(b, lane);
    }
    if (r.live) out[base[r.bucket] + mine[r.bucket] + r.rank] = (int32_t)(i0 + st + r.src);
    __syncwarp();
    if (r.live && r.last) mine[r.bucket] = (uint16_t)(mine[r.bucket] + r.len);
    __syncwarp();
  }
}

bool warp_path(const lsh_problem& p) { return p.n_buckets <= kWarpMaxBuckets; }

}  // namespace

size_t sort_ws_bytes(const lsh_problem& p) {
  const int64_t S = (int64_t)p.B * p.H * p.n_rounds;
  if (warp_path(p))
    return align_up((size_t)S * warp_geo(p).Q * p.n_buckets * 4, 256) +
           align_up((size_t)S * p.n_buckets * 4, 256);
  const int64_t tiles = (p.L + kTile - 1) / kTile;
  size_t b = align_up((size_t)S * p.L * 4, 256);
  b += align_up((size_t)S * p.n_buckets * tiles * 4, 256);
  b += align_up((size_t)S * p.n_buckets * 4, 256);
  return b;
}

SortWs sort_ws_carve(const lsh_problem& p, void* ws) {
  const int64_t S = (int64_t)p.B * p.H * p.n_rounds;
  SortWs w;
  char* c = (char*)ws;
  if (warp_path(p)) {
    w.sorted = nullptr;
    w.counts = (int32_t*)c;
    w.base = (int32_t*)(c + align_up((size_t)S * warp_geo(p).Q * p.n_buckets * 4, 256));
    return w;
  }
  const int64_t tiles = (p.L + kTile - 1) / kTile;
  w.sorted = (uint32_t*)c;
  c += align_up((size_t)S * p.L * 4, 256);
  w.counts = (int32_t*)c;
  c += align_up((size_t)S * p.n_buckets * tiles * 4, 256);
  w.base = (int32_t*)c;
  return w;
}

cudaError_t launch_sort(const lsh_problem& p, const int32_t* bucket, int32_t* perm,
                        const SortWs& ws, int* status, cudaStream_t s) {
  const int64_t S = (int64_t)p.B * p.H * p.n_rounds;
  const int64_t rows = S * p.n_buckets;
  if (warp_path(p)) {
    const WarpGeo g = warp_geo(p);
    const size_t sm_count_k = (size_t)p.n_buckets * 4;
    cudaError_t e = cudaFuncSetAttribute(sort_count_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_count_k);
    if (e != cudaSuccess) return e;
    const size_t key_bytes = (size_t)g.W * g.PW * 4;
    const bool cache = g.smem + key_bytes <= (size_t)kSortSmemBudget;
    auto scatter = cache ? sort_scatter_kernel<true> : sort_scatter_kernel<false>;
    const size_t sm_scatter = cache ? g.smem + key_bytes : g.smem;
    e = cudaFuncSetAttribute(scatter, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sm_scatter);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)(S * g.Q);
    sort_count_kernel<<<grid, 1024, sm_count_k, s>>>(bucket, ws.counts, p.L, p.n_buckets, g.P,
                                                     g.Q, status);
    if (g.scanned) {
      sort_qscan_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, s>>>(ws.counts, ws.base,
                                                                       p.n_buckets, g.Q, rows);
      sort_bscan_kernel<<<(unsigned)S, 1024, 0, s>>>(ws.base, p.n_buckets);
    }
    scatter<<<grid, g.W * 32, sm_scatter, s>>>(bucket, ws.counts,
                                                       g.scanned ? ws.base : nullptr, perm, p.L,
                                                       p.n_buckets, g.PW, g.P, g.Q);
    note_launch(g.scanned ? 4 : 2);
    return cudaGetLastError();
  }
  const int tiles = (p.L + kTile - 1) / kTile;
  cudaError_t e = cudaMemsetAsync(ws.counts, 0, (size_t)rows * tiles * 4, s);
  if (e != cudaSuccess) return e;
  tile_sort_kernel<<<(unsigned)(S * tiles), kTileThreads, 0, s>>>(bucket, ws.sorted, ws.counts, p.L,
                                                               p.n_buckets, tiles, status);
  row_scan_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(ws.counts, ws.base, rows, tiles);
  bucket_scan_kernel<<<(unsigned)S, 1024, 0, s>>>(ws.base, p.n_buckets);
  scatter_kernel<<<(unsigned)(S * tiles), kTileThreads, 0, s>>>(ws.sorted, ws.counts, ws.base, perm,
                                                             p.L, p.n_buckets, tiles);
  note_launch(4);
  return cudaGetLastError();
}

}  // namespace lsh

// ----------------------------------------------------------------------------
// Sort with library-owned scratch, for callers that cannot hand the library a
// workspace (see lsh_sort_noalloc in lsh.h).
// ----------------------------------------------------------------------------
#include <mutex>

namespace lsh {
namespace {

// Shared scratch for every lsh_sort_noalloc call on a device. Each GPU that
// loads the library holds these bytes until the process exits.
static __device__ __align__(256) unsigned char g_sort_scratch[LSH_SORT_NOALLOC_SCRATCH_BYTES];

constexpr int kScratchDevices = 64;
void* g_sort_scratch_addr[kScratchDevices] = {};
std::mutex g_sort_scratch_mu;

// Device address of g_sort_scratch on the current device. The host-side name
// of the array is only a stand-in, so the address is looked up once per
// device with that device current, and cached.
cudaError_t sort_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kScratchDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_sort_scratch_mu);
  if (!g_sort_scratch_addr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_sort_scratch);
    if (e != cudaSuccess) return e;
    g_sort_scratch_addr[dev] = ptr;
  }
  *out = g_sort_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace lsh

extern "C" lsh_status lsh_sort_noalloc(const lsh_problem* p, const int32_t* bucket, int32_t* perm,
                                       lsh_stream_t stream) {
  // Invalid and empty problems report a zero workspace size; lsh_sort then
  // returns their status without touching the device.
  const size_t need = lsh_sort_workspace_size(p);
  if (need == 0) return lsh_sort(p, bucket, perm, nullptr, 0, stream);
  if (need > (size_t)LSH_SORT_NOALLOC_SCRATCH_BYTES) return LSH_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (lsh::sort_scratch_address(&scratch) != cudaSuccess) return LSH_ERR_CUDA;
  // lsh_sort clears the per-tile counters it needs on the stream before use;
  // everything else in the scratch is overwritten.
  return lsh_sort(p, bucket, perm, scratch, (size_t)LSH_SORT_NOALLOC_SCRATCH_BYTES, stream);
}
