// topk.cu -- per-query-block top-k of the block score matrix.
//
// Speed3R (gist.science summary, "Methodologie" §1 "Selectie-tak"): the selection branch attends
// to the top-k blocks chosen by the compression branch's scores. Ties go to the lower block index.
//
// Two kernels. For k <= kWarpTopkMax (256), topk_warp_kernel streams each row once through one
// warp (see there). Larger k use topk_kernel:
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
// with a grid stride, no block-wide barrier. The warp reads its row once with 16-byte loads
// (kVec per lane of the next batch in flight while the current batch is examined) and keeps, in
// its slice of shared memory:
//   top[0, K2)   the K2 (power of two >= k) largest keys seen so far, sorted descending, zero-filled
//                while fewer than K2 keys have been seen (zero is below every real key)
//   cand[0, C)   keys appended since top was last brought up to date, unsorted
// theta = top[k-1] is the k-th largest key among those seen (or zero): at least k elements reach
// it, so an element whose key is below it cannot be in the top-k. A 32-bit compare of the score
// bits against the upper half of theta rejects almost every element once theta has risen; the few
// that pass are appended to cand by ballot. When cand would overflow, it is sorted descending and
// merged into top: the element-wise maximum of top[i] and cand[K2-1-i] holds the K2 largest keys
// of both as a bitonic sequence, which K2's half-cleaner stages sort (a warp-synchronous bitonic
// network; every compare-exchange is unrolled at compile time). At the end of the row the last
// candidates are merged the same way and top[0, k) is the row's top-k, in descending order.
// ------------------------------------------------------------------------------------------
constexpr int kRowsPerCta = 8;
#ifndef S3R_TOPK_VEC
#define S3R_TOPK_VEC 2
#endif
#ifndef S3R_TOPK_MIN_CTAS
#define S3R_TOPK_MIN_CTAS 4
#endif
constexpr int kVec = S3R_TOPK_VEC;  // 16-byte loads per lane in flight beside the current ones
constexpr int kWarpTopkMax = 256;   // K2 <= 256

__device__ __forceinline__ void cmp_exchange_desc(uint64_t* b, int e, int partner, bool desc) {
  const uint64_t x = b[e], y = b[partner];
  const uint64_t hi = x > y ? x : y, lo = x > y ? y : x;
  b[e] = desc ? hi : lo;
  b[partner] = desc ? lo : hi;
}

// descending bitonic sort of b[0, N) by one warp (N a power of two, 32 <= N)
template <int N>
__device__ __forceinline__ void warp_sort_desc(uint64_t* b, int lane) {
  constexpr int kPairs = N / 2 > 32 ? N / 64 : 1;  // compare-exchanges per lane and stage
#pragma unroll
  for (int size = 2; size <= N; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
      for (int q = 0; q < kPairs; ++q) {
        const int i = q * 32 + lane;  // pair i: element e has the stride bit clear
        if (N / 2 >= 32 || i < N / 2) {
          const int e = ((i & ~(stride - 1)) << 1) | (i & (stride - 1));
          cmp_exchange_desc(b, e, e + stride, (e & size) == 0);
        }
      }
      __syncwarp();
    }
  }
}

// sort the bitonic sequence b[0, N) descending: the half-cleaner stages of a bitonic network
template <int N>
__device__ __forceinline__ void warp_bitonic_clean_desc(uint64_t* b, int lane) {
  constexpr int kPairs = N / 2 > 32 ? N / 64 : 1;
#pragma unroll
  for (int stride = N >> 1; stride > 0; stride >>= 1) {
#pragma unroll
    for (int q = 0; q < kPairs; ++q) {
      const int i = q * 32 + lane;
      if (N / 2 >= 32 || i < N / 2) {
        const int e = ((i & ~(stride - 1)) << 1) | (i & (stride - 1));
        cmp_exchange_desc(b, e, e + stride, true);
      }
    }
    __syncwarp();
  }
}

// merge cand[0, cnt) into top (see above); returns the new theta
template <int K2, int C>
__device__ __forceinline__ uint64_t warp_merge(uint64_t* top, uint64_t* cand, int cnt, int k) {
  // the lane index is re-read here so that the compiler does not keep the unrolled networks'
  // addresses live in registers across the whole scan
  int lane;
  asm volatile("mov.u32 %0, %%laneid;\n" : "=r"(lane));
  for (int e = cnt + lane; e < C; e += 32) cand[e] = 0ull;
  __syncwarp();
  warp_sort_desc<C>(cand, lane);
  constexpr int kLo = K2 > C ? K2 - C : 0;  // below kLo, cand[K2-1-i] does not exist
#pragma unroll
  for (int i = kLo + lane; i < K2; i += 32) {
    const uint64_t x = top[i], y = cand[K2 - 1 - i];
    top[i] = x > y ? x : y;
  }
  __syncwarp();
  warp_bitonic_clean_desc<K2>(top, lane);
  return top[k - 1];
}

// The merge is inlined at each of its call sites, except for the largest list: there its
// unrolled networks are long enough that one shared copy, reached by a call, runs faster.
template <int K2, int C>
__device__ __noinline__ uint64_t warp_merge_call(uint64_t* top, uint64_t* cand, int cnt, int k) {
  return warp_merge<K2, C>(top, cand, cnt, k);
}
template <int K2, int C>
__device__ __forceinline__ uint64_t merge(uint64_t* top, uint64_t* cand, int cnt, int k) {
  if constexpr (K2 >= 256)
    return warp_merge_call<K2, C>(top, cand, cnt, k);
  else
    return warp_merge<K2, C>(top, cand, cnt, k);
}

template <int K2, int C>
__global__ void __launch_bounds__(kRowsPerCta * 32, S3R_TOPK_MIN_CTAS)
    topk_warp_kernel(const float* __restrict__ scores, int32_t* __restrict__ idx, int row_len,
                     int first, int k, int64_t rows) {
  extern __shared__ uint64_t warp_keys[];  // [kRowsPerCta][K2 + C]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* top = warp_keys + warp * (K2 + C);
  uint64_t* cand = top + K2;
  const int n = row_len - first;  // blocks first .. row_len-1 compete
  const uint32_t below = (1u << lane) - 1u;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * kRowsPerCta + warp; row < rows;
       row += static_cast<int64_t>(gridDim.x) * kRowsPerCta) {
    const uint32_t* src = reinterpret_cast<const uint32_t*>(scores + row * row_len + first);
    int32_t* out = idx + row * (first + k);
    for (int f = lane; f < first; f += 32) out[f] = f;
    out += first;
#pragma unroll
    for (int i = lane; i < K2; i += 32) top[i] = 0ull;
    __syncwarp();
    uint64_t theta = 0ull;
    int cnt = 0;
    // offer one element per lane (block index j, valid or not) to cand
    auto offer = [&](uint32_t x, int j, bool pass) {
      const uint64_t key =
          (static_cast<uint64_t>(x) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(j));
      pass = pass && key > theta;
      uint32_t m = __ballot_sync(0xffffffffu, pass);
      if (cnt + __popc(m) > C) {
        theta = merge<K2, C>(top, cand, cnt, k);
        cnt = 0;
        pass = pass && key > theta;
        m = __ballot_sync(0xffffffffu, pass);
      }
      if (pass) cand[cnt + __popc(m & below)] = key;
      cnt += __popc(m);
    };
    // offer the four elements of one 16-byte load per lane (blocks j0 .. j0+3): four exact tests,
    // a prefix count of the passing keys from three ballots (a lane passes at most four), and
    // predicated appends. If they would overflow cand, they go in one element at a time instead,
    // merging as needed.
    auto offer4 = [&](const uint4 c, const int j0, const bool v) {
      const uint32_t lo = ~static_cast<uint32_t>(j0);  // ~(j0 + e) = lo - e
      const uint64_t k0 = static_cast<uint64_t>(c.x) << 32 | lo;
      const uint64_t k1 = static_cast<uint64_t>(c.y) << 32 | (lo - 1u);
      const uint64_t k2 = static_cast<uint64_t>(c.z) << 32 | (lo - 2u);
      const uint64_t k3 = static_cast<uint64_t>(c.w) << 32 | (lo - 3u);
      const bool p0 = v && k0 > theta, p1 = v && k1 > theta, p2 = v && k2 > theta,
                 p3 = v && k3 > theta;
      const int pc = p0 + p1 + p2 + p3;
      const uint32_t b0 = __ballot_sync(0xffffffffu, pc & 1);
      const uint32_t b1 = __ballot_sync(0xffffffffu, pc & 2);
      const uint32_t b2 = __ballot_sync(0xffffffffu, pc & 4);
      const int total = __popc(b0) + 2 * __popc(b1) + 4 * __popc(b2);
      if (cnt + total > C) {
        uint4 r = c;
        uint32_t pm = p0 | p1 << 1 | p2 << 2 | p3 << 3;
#pragma unroll 1
        for (int e = 0; e < 4; ++e) {  // one copy of the code for the four elements
          offer(r.x, j0 + e, pm & 1u);
          r = make_uint4(r.y, r.z, r.w, 0u);
          pm >>= 1;
        }
        return;
      }
      int pos = cnt + __popc(b0 & below) + 2 * __popc(b1 & below) + 4 * __popc(b2 & below);
      if (p0) cand[pos++] = k0;
      if (p1) cand[pos++] = k1;
      if (p2) cand[pos++] = k2;
      if (p3) cand[pos] = k3;
      cnt += total;
    };
    // elements before the first 16-byte boundary of the row, and after the last one
    int head = static_cast<int>(((16u - (reinterpret_cast<uintptr_t>(src) & 15u)) & 15u) >> 2);
    if (head > n) head = n;
    const int nvec = (n - head) >> 2, tail0 = head + 4 * nvec;
    {
      const bool v = lane < head;
      const uint32_t x = v ? __ldg(src + lane) : 0u;
      if (__any_sync(0xffffffffu, v)) offer(x, lane, v);
    }
    const uint4* vsrc = reinterpret_cast<const uint4*>(src + head);
    uint4 x[kVec];
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
      const int vi = u * 32 + lane;
      x[u] = vi < nvec ? __ldg(vsrc + vi) : make_uint4(0u, 0u, 0u, 0u);
    }
    for (int vb = 0; vb < nvec; vb += 32 * kVec) {
#pragma unroll
      for (int u = 0; u < kVec; ++u) {
        const uint4 c = x[u];
        {  // the same slot of the next batch goes in flight before this one is examined
          const int vi = vb + 32 * kVec + u * 32 + lane;
          x[u] = vi < nvec ? __ldg(vsrc + vi) : make_uint4(0u, 0u, 0u, 0u);
        }
        const int vi = vb + u * 32 + lane;
        const bool v = vi < nvec;
        // keys with score bits below theta's upper half are below theta
        const uint32_t th = static_cast<uint32_t>(theta >> 32);
        const uint32_t mx = max(max(c.x, c.y), max(c.z, c.w));
        if (__any_sync(0xffffffffu, v && mx >= th)) offer4(c, head + 4 * vi, v);
      }
    }
    {
      const bool v = tail0 + lane < n;
      const uint32_t xt = v ? __ldg(src + tail0 + lane) : 0u;
      if (__any_sync(0xffffffffu, v)) offer(xt, tail0 + lane, v);
    }
    merge<K2, C>(top, cand, cnt, k);
    for (int e = lane; e < k; e += 32)
      out[e] = first + static_cast<int32_t>(~static_cast<uint32_t>(top[e] & 0xFFFFFFFFull));
    __syncwarp();  // the buffers are reused by the warp's next row
  }
}

template <int K2, int C>
cudaError_t launch_warp_topk(const Problem& p, const float* scores, int32_t* idx, int64_t rows,
                             cudaStream_t st) {
  constexpr int smem = kRowsPerCta * (K2 + C) * 8;
  cudaError_t e = cudaFuncSetAttribute(topk_warp_kernel<K2, C>,
                                       cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, per_sm = 1;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, topk_warp_kernel<K2, C>,
                                                         kRowsPerCta * 32, smem)) != cudaSuccess)
    return e;
  const int64_t need = (rows + kRowsPerCta - 1) / kRowsPerCta;
  const int64_t fill = static_cast<int64_t>(sms) * (per_sm > 0 ? per_sm : 1);
  const unsigned grid = static_cast<unsigned>(need < fill ? need : fill);
  topk_warp_kernel<K2, C><<<grid, kRowsPerCta * 32, smem, st>>>(
      scores, idx, static_cast<int>(p.nb), p.F, p.k, rows);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

static_assert(kWarps * 256 * 4 >= kSortMax * 8, "sort buffer must fit in the histogram space");

size_t topk_smem_bytes(int64_t nb) {
  return static_cast<size_t>(kWarps) * 256 * 4 + static_cast<size_t>(nb) * 4;
}

cudaError_t launch_topk(const Problem& p, const float* scores, int32_t* idx, cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(p.H) * p.nqb;
  if (p.k <= kWarpTopkMax) {
    if (p.k <= 32) return launch_warp_topk<32, 64>(p, scores, idx, rows, st);
    if (p.k <= 64) return launch_warp_topk<64, 64>(p, scores, idx, rows, st);
    if (p.k <= 128) return launch_warp_topk<128, 64>(p, scores, idx, rows, st);
    return launch_warp_topk<256, 128>(p, scores, idx, rows, st);
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
