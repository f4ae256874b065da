// topk.cu -- per-query-block top-k of the block score matrix.
//
// Speed3R (gist.science summary, "Methodologie" §1 "Selectie-tak"): the selection branch attends
// to the top-k blocks chosen by the compression branch's scores. Ties go to the lower block index.
//
// Two kernels. For k <= kWarpTopkMax (every default configuration), topk_warp_kernel streams each
// row once through one warp (see there). Larger k use topk_kernel:
// One CTA per score row [nb] (one query block of one head). Scores are probabilities summed over
// rows, so they are non-negative and their fp32 bit patterns order like unsigned integers; the
// 64-bit key (bits << 32 | ~index) orders by descending score, then ascending index, and is unique.
// The row is staged once in shared memory (the only HBM read: nb * 4 bytes) while every thread
// keeps the maximum of the elements it loaded.
//
// Fast path (k <= kFilterMax): the k-th largest of the 512 per-thread maxima, T0, is a lower bound
// of the k-th largest score (k distinct elements reach it), so the exact top-k is contained in the
// candidates {score >= T0}, which for non-degenerate rows number little more than k. They are
// compacted with warp-aggregated atomics and bitonic-sorted on the 64-bit key; the first k win.
//
// Exact fallback (larger k, or more than kSortMax candidates, e.g. rows of equal scores): a radix
// select finds the k-th largest pattern T in four 8-bit passes (per-warp histograms with
// warp-aggregated increments, a block scan over the 256 bins). Every element above T is taken, and
// of the elements equal to T the lowest indices, found by an in-order block prefix count. For
// k <= kSortMax the winners are bitonic-sorted as above; larger k are emitted in ascending index
// order.
// With F forced blocks (the VGGT variant's always-kept reference frame) the list opens with
// blocks 0 .. F-1 and the top-k runs over the rest of the row only.
#include "common.cuh"
#include "internal.h"

namespace s3r {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kSortMax = 2048;   // largest k whose output is sorted; also the candidate cap
constexpr int kFilterMax = 512;  // largest k for the threshold-filter fast path (= kThreads)

// descending bitonic sort of n keys (n a power of two) in shared memory; all threads call it
template <typename T>
__device__ __forceinline__ void bitonic_sort_desc(T* a, int n) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int e = threadIdx.x; e < n; e += kThreads) {
        const int partner = e ^ stride;
        if (partner > e) {
          const bool desc = (e & size) == 0;
          const T x = a[e], y = a[partner];
          if ((x < y) == desc) {
            a[e] = y;
            a[partner] = x;
          }
        }
      }
      __syncthreads();
    }
  }
}

// exclusive prefix sum over the block of one int per thread, in thread order; returns the total
__device__ __forceinline__ int block_exclusive_scan(int x, int* warp_sums, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kWarps ? warp_sums[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    if (lane < kWarps) warp_sums[lane] = wi - w;  // exclusive warp offsets
    if (lane == kWarps - 1) warp_sums[kWarps] = wi;
  }
  __syncthreads();
  const int res = warp_sums[warp] + incl - x;
  total = warp_sums[kWarps];
  __syncthreads();  // warp_sums may be reused right away
  return res;
}

__global__ void __launch_bounds__(kThreads)
    topk_kernel(const float* __restrict__ scores, int32_t* __restrict__ idx, int row_len,
                int first, int k) {
  // dynamic shared memory: [kWarps][256] histograms (reused as the sort buffer), then [nb] keys
  extern __shared__ __align__(16) uint32_t smem_dyn[];
  int(*hist)[256] = reinterpret_cast<int(*)[256]>(smem_dyn);
  uint32_t* sm_keys = smem_dyn + kWarps * 256;
  __shared__ int warp_sums[kWarps + 1];
  __shared__ uint32_t s_prefix;
  __shared__ int s_kk;
  __shared__ uint32_t s_max[kThreads];
  __shared__ int s_count;

  // blocks 0 .. first-1 open the list without competing; the top-k ranks the other nb of the row
  const int nb = row_len - first;
  const int64_t row = blockIdx.x;
  const uint32_t* src = reinterpret_cast<const uint32_t*>(scores + row * row_len + first);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int32_t* out = idx + row * (first + k);
  for (int f = tid; f < first; f += kThreads) out[f] = f;
  out += first;
  uint64_t* sort_buf = reinterpret_cast<uint64_t*>(smem_dyn);  // aliases the histograms

  uint32_t my_max = 0;
  {
    int j = tid;
    for (; j + 3 * kThreads < nb; j += 4 * kThreads) {  // 4 loads in flight per thread
      uint32_t x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) x[u] = __ldg(src + j + u * kThreads);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        sm_keys[j + u * kThreads] = x[u];
        my_max = max(my_max, x[u]);
      }
    }
    for (; j < nb; j += kThreads) {
      const uint32_t x = __ldg(src + j);
      sm_keys[j] = x;
      my_max = max(my_max, x);
    }
  }
  s_max[tid] = my_max;  // threads that loaded nothing contribute 0, below every candidate used
  if (tid == 0) {
    s_prefix = 0;
    s_kk = k;
    s_count = 0;
  }
  __syncthreads();

  if (k <= kFilterMax && k <= nb) {
    bitonic_sort_desc(s_max, kThreads);
    const uint32_t t0 = s_max[k - 1];
    // at least k elements are >= t0 (the k largest per-thread maxima are distinct elements),
    // unless fewer than k threads loaded anything; then t0 = 0 and every element qualifies
    for (int j0 = 0; j0 < nb; j0 += kThreads) {
      const int j = j0 + tid;
      const bool cand = j < nb && sm_keys[j < nb ? j : 0] >= t0;
      const uint32_t m = __ballot_sync(0xffffffffu, cand);
      int base = 0;
      if (lane == 0 && m) base = atomicAdd(&s_count, __popc(m));
      base = __shfl_sync(0xffffffffu, base, 0);
      if (cand) {
        const int pos = base + __popc(m & ((1u << lane) - 1u));
        if (pos < kSortMax)
          sort_buf[pos] = (static_cast<uint64_t>(sm_keys[j]) << 32) |
                          static_cast<uint32_t>(~static_cast<uint32_t>(j));
      }
    }
    __syncthreads();
    const int count = s_count;
    if (count <= kSortMax) {
      int n2 = 1;
      while (n2 < count) n2 <<= 1;
      for (int e = count + tid; e < n2; e += kThreads) sort_buf[e] = 0ull;
      __syncthreads();
      bitonic_sort_desc(sort_buf, n2);
      for (int e = tid; e < k; e += kThreads)
        out[e] = first + static_cast<int32_t>(~static_cast<uint32_t>(sort_buf[e] & 0xFFFFFFFFull));
      return;
    }
    // too many candidates (degenerate row): fall through to the exact radix select
  }

  uint32_t mask = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = tid; b < kWarps * 256; b += kThreads) (&hist[0][0])[b] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix;
    for (int j0 = 0; j0 < nb; j0 += kThreads) {
      const int j = j0 + tid;
      const bool in = j < nb && (sm_keys[j < nb ? j : 0] & mask) == prefix;
      const uint32_t digit = in ? (sm_keys[j] >> shift) & 0xFFu : 0x100u + lane;  // unique if out
      const uint32_t peers = __match_any_sync(0xffffffffu, digit);
      if (in && (__ffs(peers) - 1) == lane) atomicAdd(&hist[warp][digit], __popc(peers));
    }
    __syncthreads();
    // bins in descending digit order: thread t < 256 owns digit 255 - t
    int cnt = 0;
    if (tid < 256) {
      const int dgt = 255 - tid;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) cnt += hist[w][dgt];
    }
    int total;
    const int before = block_exclusive_scan(tid < 256 ? cnt : 0, warp_sums, total);
    const int kk = s_kk;
    __syncthreads();
    if (tid < 256 && before < kk && kk <= before + cnt) {
      s_prefix = prefix | (static_cast<uint32_t>(255 - tid) << shift);
      s_kk = kk - before;
    }
    mask |= 0xFFu << shift;
    __syncthreads();
  }
  const uint32_t T = s_prefix;  // bits of the k-th largest score
  const int take_eq = s_kk;     // how many of the elements equal to T are selected

  // in-order compaction: all elements > T, the first take_eq elements == T
  const bool sorted_out = k <= kSortMax;
  int eq_base = 0, out_base = 0;
  for (int j0 = 0; j0 < nb; j0 += kThreads) {
    const int j = j0 + tid;
    const uint32_t u = j < nb ? sm_keys[j] : 0u;
    const bool gt = j < nb && u > T;
    const bool eq = j < nb && u == T;
    int eq_total;
    const int eq_rank = eq_base + block_exclusive_scan(eq ? 1 : 0, warp_sums, eq_total);
    const bool take = gt || (eq && eq_rank < take_eq);
    int take_total;
    const int pos = out_base + block_exclusive_scan(take ? 1 : 0, warp_sums, take_total);
    if (take) {
      if (sorted_out)
        sort_buf[pos] = (static_cast<uint64_t>(u) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(j));
      else
        out[pos] = first + j;
    }
    eq_base += eq_total;
    out_base += take_total;
  }
  if (!sorted_out) return;

  int n2 = 1;
  while (n2 < k) n2 <<= 1;
  for (int e = k + tid; e < n2; e += kThreads) sort_buf[e] = 0ull;  // below every real key
  __syncthreads();
  bitonic_sort_desc(sort_buf, n2);
  for (int e = tid; e < k; e += kThreads)
    out[e] = first + static_cast<int32_t>(~static_cast<uint32_t>(sort_buf[e] & 0xFFFFFFFFull));
}

// ------------------------------------------------------------------------------------------
// Streaming path for k <= kWarpTopkMax: one warp per row, kRowsPerCta warps per CTA walking rows
// with a grid stride, no block-wide barrier. The warp reads its row once with coalesced loads
// (the next kUnroll per lane in flight while the current ones are examined) and keeps in shared
// memory a buffer of candidate keys together with theta, the k-th largest key among those it has
// dropped or kept so far: at least k elements have keys >= theta, so an element whose key is
// below it cannot be in the top-k. A 32-bit compare of the score bits against the upper half of
// theta rejects almost every element once theta has risen; the few that pass are appended by
// ballot. When the buffer would overflow it is sorted (warp-synchronous bitonic sort, descending)
// and cut to its first k keys, and theta becomes the k-th. At the end of the row the buffer is
// sorted once more and its first k keys are the row's top-k, in descending order. The buffer
// holds kCap >= 2k + 32 keys, so a cut frees room for at least k + 32 more.
// ------------------------------------------------------------------------------------------
constexpr int kRowsPerCta = 8;
#ifndef S3R_TOPK_UNROLL
#define S3R_TOPK_UNROLL 8
#endif
#ifndef S3R_TOPK_MIN_CTAS
#define S3R_TOPK_MIN_CTAS 4
#endif
constexpr int kUnroll = S3R_TOPK_UNROLL;  // loads per lane in flight beside the current ones
constexpr int kWarpTopkMax = 240;  // 2k + 32 <= 512

// descending bitonic sort of buf[0, n) by one warp; n a power of two, 32 <= n
__device__ __forceinline__ void warp_bitonic_desc(uint64_t* buf, int n, int lane) {
  for (int lsize = 1; (1 << lsize) <= n; ++lsize) {
    const int size = 1 << lsize;
    for (int lst = lsize - 1; lst >= 0; --lst) {
      const int stride = 1 << lst;
      for (int i = lane; i < (n >> 1); i += 32) {  // pair i: e has bit lst clear
        const int e = ((i >> lst) << (lst + 1)) | (i & (stride - 1)), partner = e + stride;
        const bool desc = (e & size) == 0;
        const uint64_t x = buf[e], y = buf[partner];
        if ((x < y) == desc) {
          buf[e] = y;
          buf[partner] = x;
        }
      }
      __syncwarp();
    }
  }
}

// sort the warp's cnt candidates and keep the first min(k, cnt); returns the new count and sets
// theta to the k-th key (0 while fewer than k candidates exist)
__device__ __forceinline__ int warp_compact(uint64_t* buf, int cnt, int k, uint64_t& theta,
                                            int lane) {
  int n2 = 32;
  while (n2 < cnt) n2 <<= 1;
  for (int e = cnt + lane; e < n2; e += 32) buf[e] = 0ull;  // below every real key
  __syncwarp();
  warp_bitonic_desc(buf, n2, lane);
  const int kept = cnt < k ? cnt : k;
  theta = cnt >= k ? buf[k - 1] : 0ull;
  __syncwarp();
  return kept;
}

template <int kCap>
__global__ void __launch_bounds__(kRowsPerCta * 32, S3R_TOPK_MIN_CTAS)
    topk_warp_kernel(const float* __restrict__ scores, int32_t* __restrict__ idx, int row_len,
                     int first, int k, int64_t rows) {
  extern __shared__ uint64_t warp_keys[];  // [kRowsPerCta][kCap]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* buf = warp_keys + warp * kCap;
  const int n = row_len - first;  // blocks first .. row_len-1 compete
  const uint32_t below = (1u << lane) - 1u;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * kRowsPerCta + warp; row < rows;
       row += static_cast<int64_t>(gridDim.x) * kRowsPerCta) {
    const uint32_t* src = reinterpret_cast<const uint32_t*>(scores + row * row_len + first);
    int32_t* out = idx + row * (first + k);
    for (int f = lane; f < first; f += 32) out[f] = f;
    out += first;
    uint64_t theta = 0ull;
    int cnt = 0;
    uint32_t x[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int j = u * 32 + lane;
      x[u] = j < n ? __ldg(src + j) : 0u;
    }
    for (int base = 0; base < n; base += 32 * kUnroll) {
      uint32_t nx[kUnroll];  // the next batch, in flight while this one is examined
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int j = base + 32 * kUnroll + u * 32 + lane;
        nx[u] = j < n ? __ldg(src + j) : 0u;
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int j = base + u * 32 + lane;
        // keys with score bits below theta's upper half are below theta
        bool pass = j < n && x[u] >= static_cast<uint32_t>(theta >> 32);
        if (!__any_sync(0xffffffffu, pass)) continue;
        const uint64_t key = (static_cast<uint64_t>(x[u]) << 32) |
                             static_cast<uint32_t>(~static_cast<uint32_t>(j));
        pass = pass && key > theta;
        uint32_t m = __ballot_sync(0xffffffffu, pass);
        if (cnt + __popc(m) > kCap) {
          cnt = warp_compact(buf, cnt, k, theta, lane);
          pass = pass && key > theta;
          m = __ballot_sync(0xffffffffu, pass);
        }
        if (pass) buf[cnt + __popc(m & below)] = key;
        cnt += __popc(m);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) x[u] = nx[u];
    }
    __syncwarp();
    cnt = warp_compact(buf, cnt, k, theta, lane);
    for (int e = lane; e < k; e += 32)
      out[e] = first + static_cast<int32_t>(~static_cast<uint32_t>(buf[e] & 0xFFFFFFFFull));
    __syncwarp();  // the buffer is reused by the warp's next row
  }
}

template <int kCap>
cudaError_t launch_warp_topk(const Problem& p, const float* scores, int32_t* idx, int64_t rows,
                             cudaStream_t st) {
  constexpr int smem = kRowsPerCta * kCap * 8;
  cudaError_t e = cudaFuncSetAttribute(topk_warp_kernel<kCap>,
                                       cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, per_sm = 1;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, topk_warp_kernel<kCap>,
                                                         kRowsPerCta * 32, smem)) != cudaSuccess)
    return e;
  const int64_t need = (rows + kRowsPerCta - 1) / kRowsPerCta;
  const int64_t fill = static_cast<int64_t>(sms) * (per_sm > 0 ? per_sm : 1);
  const unsigned grid = static_cast<unsigned>(need < fill ? need : fill);
  topk_warp_kernel<kCap><<<grid, kRowsPerCta * 32, smem, st>>>(
      scores, idx, static_cast<int>(p.nb), p.F, p.k, rows);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

static_assert(kWarps * 256 * 4 >= kSortMax * 8, "sort buffer must fit in the histogram space");
static_assert(2 * kWarpTopkMax + 32 <= 512, "the largest buffer holds 2k + 32 keys");

size_t topk_smem_bytes(int64_t nb) {
  return static_cast<size_t>(kWarps) * 256 * 4 + static_cast<size_t>(nb) * 4;
}

cudaError_t launch_topk(const Problem& p, const float* scores, int32_t* idx, cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(p.H) * p.nqb;
  if (p.k <= kWarpTopkMax) {
    if (2 * p.k + 32 <= 128) return launch_warp_topk<128>(p, scores, idx, rows, st);
    if (2 * p.k + 32 <= 256) return launch_warp_topk<256>(p, scores, idx, rows, st);
    return launch_warp_topk<512>(p, scores, idx, rows, st);
  }
  const size_t smem = topk_smem_bytes(p.nb);
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  topk_kernel<<<static_cast<unsigned>(rows), kThreads, smem, st>>>(scores, idx,
                                                                   static_cast<int>(p.nb), p.F, p.k);
  count_launch();
  return cudaGetLastError();
}

}  // namespace s3r
