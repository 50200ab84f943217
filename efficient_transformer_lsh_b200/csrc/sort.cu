// Stable sort of positions by bucket, one segment per (batch, head, round).
//
// "Reformer: The Efficient Transformer" (research.elamur.ai summary page),
// Summary and Key points "LSH attention": positions are sorted by bucket
// before chunking. Sorting stably by bucket is sorting by the packed key
// (round, bucket, position), because positions arrive in increasing order.
//
// Counting sort in four passes over tiles of positions:
//   1. per tile, how many positions of each bucket it holds:
//      counts[seg][bucket][tile]. For n_buckets <= 4096 (tiles of 2048) a
//      warp walks 256 consecutive positions 32 at a time and counts with
//      __match_any_sync into per-warp 16-bit counters; for larger bucket
//      counts (tiles of 4096) the tile's packed keys (bucket << 12 | local
//      index) are sorted in shared memory by a bitonic network and stored;
//   2. row_scan: for every (seg, bucket), exclusive scan over tiles, plus the
//      bucket total;
//   3. bucket_scan: for every seg, exclusive scan of bucket totals;
//   4. scatter: slot = base[seg][b] + counts[seg][b][tile] + rank of the
//      position among the tile's positions of bucket b; perm[seg][slot] =
//      position. The warp path recomputes the ranks in position order (step
//      by step, lanes in order, warps in order through an exclusive prefix
//      of the per-warp counts); the bitonic path takes them from the sorted
//      packed keys, whose local index breaks ties.
// Ranks follow position order inside a tile and tiles are placed in position
// order, so the whole sort is stable.
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
        if (status) atomicExch(status, (int)LSH_ERR_DEVICE_CHECK);
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

// ---- warp-counting path (n_buckets <= kWarpMaxBuckets) --------------------
constexpr int kWarpMaxBuckets = 4096;
constexpr int kWarpsPerTile = 8;
constexpr int kWarpKeys = 256;                        // positions per warp
constexpr int kWTile = kWarpsPerTile * kWarpKeys;     // 2048 positions per tile
constexpr size_t kWarpSmem = (size_t)kWarpsPerTile * kWarpMaxBuckets * 2 + kWarpMaxBuckets * 4;

// Counts of each bucket among this warp's 256 positions into cnt[b] (16-bit).
__device__ __forceinline__ void warp_count(const int32_t* __restrict__ src, int n, int w, int lane,
                                           uint16_t* cnt, int n_buckets, int* status) {
  for (int st = 0; st < kWarpKeys / 32; ++st) {
    const int i = w * kWarpKeys + st * 32 + lane;
    uint32_t b = 0xffffffffu;
    if (i < n) {
      b = (uint32_t)src[i];
      if (b >= (uint32_t)n_buckets) {
        if (status) atomicExch(status, (int)LSH_ERR_DEVICE_CHECK);
        b = (uint32_t)n_buckets - 1;
      }
    }
    const uint32_t peers = __match_any_sync(0xffffffffu, b);
    const int leader = __ffs(peers) - 1;
    if (i < n && lane == leader) cnt[b] = (uint16_t)(cnt[b] + __popc(peers));
    __syncwarp();
  }
}

__global__ void __launch_bounds__(kWarpsPerTile * 32)
warp_count_kernel(const int32_t* __restrict__ bucket, int32_t* __restrict__ counts, int L,
                  int n_buckets, int tiles, int* status) {
  extern __shared__ uint8_t sm[];
  uint16_t* hist = reinterpret_cast<uint16_t*>(sm);     // [warps][n_buckets]
  const int tile = blockIdx.x % tiles;
  const int64_t seg = blockIdx.x / tiles;
  const int64_t p0 = (int64_t)tile * kWTile;
  const int n = min(kWTile, (int)(L - p0));
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kWarpsPerTile * n_buckets; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  warp_count(bucket + seg * L + p0, n, w, lane, hist + w * n_buckets, n_buckets, status);
  __syncthreads();
  int32_t* out = counts + seg * n_buckets * (int64_t)tiles + tile;
  for (int b = threadIdx.x; b < n_buckets; b += blockDim.x) {
    int tot = 0;
#pragma unroll
    for (int ww = 0; ww < kWarpsPerTile; ++ww) tot += hist[ww * n_buckets + b];
    out[(int64_t)b * tiles] = tot;
  }
}

__global__ void __launch_bounds__(kWarpsPerTile * 32)
warp_scatter_kernel(const int32_t* __restrict__ bucket, const int32_t* __restrict__ counts,
                    const int32_t* __restrict__ base, int32_t* __restrict__ perm, int L,
                    int n_buckets, int tiles) {
  extern __shared__ uint8_t sm[];
  uint16_t* cnt = reinterpret_cast<uint16_t*>(sm);      // [warps][n_buckets]
  int32_t* off = reinterpret_cast<int32_t*>(sm + (size_t)kWarpsPerTile * n_buckets * 2);
  const int tile = blockIdx.x % tiles;
  const int64_t seg = blockIdx.x / tiles;
  const int64_t p0 = (int64_t)tile * kWTile;
  const int n = min(kWTile, (int)(L - p0));
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* src = bucket + seg * L + p0;
  for (int i = threadIdx.x; i < kWarpsPerTile * n_buckets; i += blockDim.x) cnt[i] = 0;
  for (int b = threadIdx.x; b < n_buckets; b += blockDim.x) {
    const int64_t row = seg * n_buckets + b;
    off[b] = base[row] + counts[row * tiles + tile];
  }
  __syncthreads();
  warp_count(src, n, w, lane, cnt + w * n_buckets, n_buckets, nullptr);
  __syncthreads();
  // exclusive prefix over warps: cnt[w][b] becomes the start of warp w's run
  for (int b = threadIdx.x; b < n_buckets; b += blockDim.x) {
    int acc = 0;
#pragma unroll
    for (int ww = 0; ww < kWarpsPerTile; ++ww) {
      const int c = cnt[ww * n_buckets + b];
      cnt[ww * n_buckets + b] = (uint16_t)acc;
      acc += c;
    }
  }
  __syncthreads();
  uint16_t* mine = cnt + w * n_buckets;
  int32_t* out = perm + seg * L;
  for (int st = 0; st < kWarpKeys / 32; ++st) {
    const int i = w * kWarpKeys + st * 32 + lane;
    uint32_t b = 0xffffffffu;
    if (i < n) {
      b = (uint32_t)src[i];
      if (b >= (uint32_t)n_buckets) b = (uint32_t)n_buckets - 1;
    }
    const uint32_t peers = __match_any_sync(0xffffffffu, b);
    const int leader = __ffs(peers) - 1;
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (i < n) out[off[b] + mine[b] + rank] = (int32_t)(p0 + i);
    __syncwarp();
    if (i < n && lane == leader) mine[b] = (uint16_t)(mine[b] + __popc(peers));
    __syncwarp();
  }
}

bool warp_path(const lsh_problem& p) { return p.n_buckets <= kWarpMaxBuckets; }

}  // namespace

size_t sort_ws_bytes(const lsh_problem& p) {
  const int64_t S = (int64_t)p.B * p.H * p.n_rounds;
  const int64_t tiles = warp_path(p) ? (p.L + kWTile - 1) / kWTile : (p.L + kTile - 1) / kTile;
  size_t b = warp_path(p) ? 0 : align_up((size_t)S * p.L * 4, 256);
  b += align_up((size_t)S * p.n_buckets * tiles * 4, 256);
  b += align_up((size_t)S * p.n_buckets * 4, 256);
  return b;
}

SortWs sort_ws_carve(const lsh_problem& p, void* ws) {
  const int64_t S = (int64_t)p.B * p.H * p.n_rounds;
  const int64_t tiles = warp_path(p) ? (p.L + kWTile - 1) / kWTile : (p.L + kTile - 1) / kTile;
  char* c = (char*)ws;
  SortWs w;
  w.sorted = warp_path(p) ? nullptr : (uint32_t*)c;
  if (!warp_path(p)) c += align_up((size_t)S * p.L * 4, 256);
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
    const int tiles = (p.L + kWTile - 1) / kWTile;
    const size_t sm = (size_t)kWarpsPerTile * p.n_buckets * 2 + (size_t)p.n_buckets * 4;
    cudaError_t e = cudaFuncSetAttribute(warp_count_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kWarpSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(warp_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kWarpSmem);
    if (e != cudaSuccess) return e;
    warp_count_kernel<<<(unsigned)(S * tiles), kWarpsPerTile * 32, sm, s>>>(bucket, ws.counts, p.L,
                                                                            p.n_buckets, tiles, status);
    row_scan_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(ws.counts, ws.base, rows, tiles);
    bucket_scan_kernel<<<(unsigned)S, 1024, 0, s>>>(ws.base, p.n_buckets);
    warp_scatter_kernel<<<(unsigned)(S * tiles), kWarpsPerTile * 32, sm, s>>>(
        bucket, ws.counts, ws.base, perm, p.L, p.n_buckets, tiles);
    note_launch(4);
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
