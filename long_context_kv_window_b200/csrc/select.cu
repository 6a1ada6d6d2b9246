// select.cu -- top-k with a forced window, and per-row attention statistics.
//
// FastKV (gist.science 2502.01068) section 2.A: the selected tokens go on
// together with the observation-window tokens; section 2.B: the TSP rate and
// the KV retention rate are independent budgets over the same scores.
// StructKV (gist.science 2604.06746) section 2.B: attention entropy, sparsity
// (here: mass of the top 1 % keys) and variance per layer.
//
// Design: one thread-block cluster per ranking row -- kCS = 8 CTAs, or
// kCSWide = 16 for a lone long row (the all-head TSP row) when the device can
// place such a cluster.  Each CTA owns a contiguous segment of the row; it
// stages the segment's row sums (a row group, e.g. the eight KV-head rows of
// the TSP ranking, is summed while staging) and keeps its pooled values in
// shared memory.  Keys are an order-preserving uint32 image of the fp32 score.
// The exact k-th largest key is found in three cluster steps:
//   1. every CTA samples its pooled keys; the cluster's sorted sample brackets
//      the k-th largest key with a key window (sample quantiles around k/L);
//   2. a 1024-bin histogram over that window (one bin below, one above) is
//      summed through distributed shared memory and gives the bin holding the
//      k-th largest key -- typically a few dozen keys, however concentrated
//      the scores are (a fixed-digit radix would see one bin hold most keys);
//   3. those candidate keys, with their positions, are gathered into every
//      CTA, which picks the threshold itself and, from the positions, knows
//      how many selected keys precede each of its warps -- the
//      order-preserving compaction (ascending positions) then needs no
//      further exchange.  Ties at the threshold go to the lowest positions.
// If the window misses (the k-th key lies outside it) or its bin holds more
// than kCandMax keys (heavy ties), a plain radix select runs cluster-wide
// instead (11 + 11 + 10 bits).
#include <cooperative_groups.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace kvc {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kCS = 8;          // CTAs per ranking row (portable cluster size)
constexpr int kCSWide = 16;     // CTAs for a lone long row (non-portable cluster size)
constexpr int64_t kWideMinKeys = 32768;  // shortest row that gets the wide cluster
constexpr int kMaxHalf = 32;    // pool_kernel <= 65
constexpr int kBins = 2048;     // radix bins of the first two passes
constexpr int kWinBins = 1024;  // bins of the windowed histogram
constexpr int kWin = kWinBins - 2;  // its interior bins (bin 0: below the window; last: above)
constexpr int kSampleTotal = 128;   // sampled keys per ranking row
constexpr int kCandMax = 1024;      // largest threshold bin resolved from a candidate list

__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t b = __float_as_uint(v);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

struct __align__(16) RadixShared {
  int hist[2][kBins];  // local histograms (alternating between passes)
  int tot[kBins];      // cluster-summed histogram
  uint32_t warp_tmp[kWarps + 1];  // [kWarps] holds the last scan's block total
  uint32_t found_bucket;
  uint32_t found_rem;
};

// Exclusive block-wide scan of one uint32 per thread (sum); every thread's
// *total receives the block total.  warp_tmp has kWarps + 1 entries.  All
// threads must call it.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* warp_tmp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();  // warp_tmp may still be read from a previous call
  if (lane == 31) warp_tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = warp_tmp[lane];
    uint32_t s = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_tmp[lane] = s - t;  // exclusive prefix of warp totals
    if (lane == 31) warp_tmp[kWarps] = s;
  }
  __syncthreads();
  *total = warp_tmp[kWarps];
  return warp_tmp[warp] + x - v;
}

// Bin of histogram h (nbins = 1024 or 2048, shared memory) that holds the
// want-th largest key: count(bins above) < want <= count(bins above) + h[bin].
// Bins are visited from the top.  Returns through sh.found_*; all threads call.
__device__ void scan_find(RadixShared& sh, const int* h, int nbins, uint32_t want) {
  // thread t owns the group of bins (kThreads-1-t): higher t = lower bins
  const int per = nbins / kThreads;  // 1 or 2
  const int grp = kThreads - 1 - threadIdx.x;
  uint32_t mine = 0;
  for (int q = 0; q < per; ++q) mine += h[grp * per + q];
  uint32_t total;
  uint32_t above = block_excl_scan(mine, sh.warp_tmp, &total);
  for (int q = per - 1; q >= 0; --q) {
    const int bin = grp * per + q;
    const uint32_t c = h[bin];
    if (above < want && want <= above + c) {
      sh.found_bucket = bin;
      sh.found_rem = want - above;
    }
    above += c;
  }
  __syncthreads();
}

// After every CTA of the cluster filled hist[buf] (and a cluster barrier),
// sum the CS histograms into tot and find the bin that holds the want-th
// largest key of the cluster (scan_find).
// 16 bytes of CTA `rank`'s shared memory at this CTA's shared address `local`.
__device__ __forceinline__ int4 ld_dsmem_v4(uint32_t local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(rank));
  int4 v;
  asm volatile("ld.shared::cluster.v4.s32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(remote)
               : "memory");
  return v;
}

template <int CS>
__device__ void cluster_find_bucket(cg::cluster_group& cluster, RadixShared& sh, int buf, int nbins,
                                    uint32_t want) {
  if constexpr (CS <= 8) {
    // 16-byte loads of every rank's histogram, all issued before the sum: one
    // round trip through distributed shared memory
    for (int v4 = threadIdx.x; v4 < nbins / 4; v4 += kThreads) {
      int4 part[CS];
      const uint32_t local = (uint32_t)__cvta_generic_to_shared(&sh.hist[buf][4 * v4]);
#pragma unroll
      for (int c = 0; c < CS; ++c) part[c] = ld_dsmem_v4(local, (uint32_t)c);
      int4 acc = part[0];
#pragma unroll
      for (int c = 1; c < CS; ++c) {
        acc.x += part[c].x;
        acc.y += part[c].y;
        acc.z += part[c].z;
        acc.w += part[c].w;
      }
      reinterpret_cast<int4*>(sh.tot)[v4] = acc;
    }
  } else {
    // Larger clusters: every rank reading every histogram moves CS^2
    // histograms through the cluster.  Instead each rank sums its own slice
    // of the bins over all ranks (a reduce-scatter), and after a cluster
    // barrier collects the CS summed slices: 2 x CS slices per rank.
    const int slice = nbins / CS;  // a multiple of 4
    const uint32_t me = cluster.block_rank();
    for (int v4 = threadIdx.x; v4 < slice / 4; v4 += kThreads) {
      const int bin = (int)me * slice + 4 * v4;
      int4 part[CS];
      const uint32_t local = (uint32_t)__cvta_generic_to_shared(&sh.hist[buf][bin]);
#pragma unroll
      for (int c = 0; c < CS; ++c) part[c] = ld_dsmem_v4(local, (uint32_t)c);
      int4 acc = part[0];
#pragma unroll
      for (int c = 1; c < CS; ++c) {
        acc.x += part[c].x;
        acc.y += part[c].y;
        acc.z += part[c].z;
        acc.w += part[c].w;
      }
      *reinterpret_cast<int4*>(&sh.tot[bin]) = acc;
    }
    cluster.sync();
    // other ranks' slices (this rank's own slice is in place); a rank writes
    // only slices it does not own, and reads only the owners' slices
    for (int v4 = threadIdx.x; v4 < nbins / 4; v4 += kThreads) {
      const uint32_t owner = (uint32_t)(4 * v4 / slice);
      if (owner == me) continue;
      const uint32_t local = (uint32_t)__cvta_generic_to_shared(&sh.tot[4 * v4]);
      reinterpret_cast<int4*>(sh.tot)[v4] = ld_dsmem_v4(local, owner);
    }
  }
  __syncthreads();
  scan_find(sh, sh.tot, nbins, want);
}

__device__ __forceinline__ uint32_t warp_sum(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Split cluster barrier: arrive once this CTA reads no other CTA's shared
// memory any more, wait before exiting (no CTA may leave while another still
// reads its shared memory).
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// --------------------------------------------------------------------------
// selection
// --------------------------------------------------------------------------
struct SelArgs {
  const float* scores;
  int64_t row_stride;
  int row_group;
  const int32_t* cu;  // nullptr: one sequence of length n
  int64_t n;
  int w;
  int pool;
  int64_t k;
  int32_t* idx;
  int64_t idx_row_stride;  // per output row (single); varlen uses k
  int32_t* counts;         // varlen only, may be nullptr
  float* vals_g;           // pooled prefix scores in global memory, or nullptr
  int64_t vals_stride;     // per output row
  bool vals_packed;        // vals_g indexed by packed token offset (varlen / workspace)
  bool smem_vals;          // keep this CTA's pooled segment in shared memory
  int64_t seg_cap;         // smem mode: longest segment the dynamic smem holds
  int v_off;               // smem mode: words of dynamic smem before the pooled values
  int out_rows;
  int32_t* err;
};

struct SelShared {
  RadixShared rx;
  uint2 cand[kCandMax];            // candidate list: (key, segment position), rank by rank
  uint32_t sample[kSampleTotal];   // this CTA's sampled keys
  uint32_t sall[kSampleTotal];     // the cluster's samples (rank order), then ...
  uint32_t ssort[kSampleTotal];    // ... sorted, largest first
  uint32_t soff[kCSWide + 1];      // sample slots per rank
  uint32_t cand_off[kCSWide + 1];  // candidate slots per rank, total last
  uint32_t cand_n;                 // candidate slots this CTA has taken
  uint32_t above;                  // this CTA's keys in bins above the threshold bin
  uint32_t T, need_eq;             // threshold resolved from the candidate list
  uint32_t cnt_gt, cnt_eq;         // plain-radix path: this CTA's keys above / equal to the threshold
  uint32_t g_prev, e_prev;         // plain-radix path: the same summed over the lower ranks
  uint32_t warp_gt[kWarps], warp_eq[kWarps];
  uint32_t red[2][kWarps];
};

// Histogram increment (shared-memory atomics; callers spread the lanes of a
// warp over distant positions, whose keys rarely share a bin).
__device__ __forceinline__ void hist_add(int* hist, uint32_t bin, bool active) {
  if (active) atomicAdd(&hist[bin], 1);
}

// Block-wide sums of two counters (all threads get both).
__device__ __forceinline__ void block_sum2(uint32_t& x, uint32_t& y, uint32_t (*red)[kWarps]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  x = warp_sum(x);
  y = warp_sum(y);
  if (lane == 0) {
    red[0][warp] = x;
    red[1][warp] = y;
  }
  __syncthreads();
  x = warp_sum(red[0][lane]);
  y = warp_sum(red[1][lane]);
  __syncthreads();
}

// Warp-wide exclusive prefix sum.
__device__ __forceinline__ uint32_t warp_excl_scan(uint32_t v) {
  const int lane = threadIdx.x & 31;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x - v;
}

// Order key of pooled value t: shared-memory mode stores the keys
// themselves, global-memory mode the fp32 sums.
struct PooledKeys {
  const uint32_t* keys;  // shared-memory mode (16-byte aligned), else nullptr
  const float* vals;     // global-memory mode
  __device__ __forceinline__ uint32_t at(int t) const { return keys ? keys[t] : order_key(vals[t]); }
  // keys of positions p .. p+3; positions at or past `end` give 0 (the caller masks them)
  __device__ __forceinline__ void four(int p, int end, uint32_t (&key)[4]) const {
    if (keys && p + 4 <= end) {
      const uint4 k4 = *reinterpret_cast<const uint4*>(keys + p);
      key[0] = k4.x;
      key[1] = k4.y;
      key[2] = k4.z;
      key[3] = k4.w;
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) key[q] = p + q < end ? at(p + q) : 0u;
    }
  }
};

// The i-th position of a 1024-position block, spread so that the lanes of a
// warp sit 32 positions apart (their keys rarely share a histogram bin).
__device__ __forceinline__ int spread_index(int warp, int lane) { return lane * 32 + ((warp + lane) & 31); }

// Dynamic shared memory of the selection kernel (words): [candidate list,
// which first holds the staged row sums of the segment plus halo][pooled
// values of the segment (smem mode)].
__host__ __device__ inline int stage_halo(int half) { return (half + 3) & ~3; }
inline size_t round4(int64_t x) { return (size_t)((x + 3) & ~int64_t(3)); }
inline size_t sel_v_words(int64_t seg) { return round4(seg) + 4; }
inline size_t sel_stage_words(int64_t seg, int half) { return round4(seg) + 2 * stage_halo(half) + 4; }
// Positions per CTA: a multiple of 4, so that segments start 16-byte aligned.
__host__ __device__ inline int64_t sel_segment(int64_t L, int cs) { return ((L + cs - 1) / cs + 3) & ~int64_t(3); }

// Row sums of `row_group` score rows over stage positions [p0, p0 + 4*n4)
// into st4, zero outside [0, L), with 16-byte loads: RU rows x PU positions
// of loads in flight per thread before any of them is summed (a row-group sum
// of eight rows then costs one round trip to L2 per position, not eight).
// Every position is summed in row order starting from +0, whatever RU is.
template <int RU, int PU>
__device__ __forceinline__ void stage_row_sums(float4* st4, int n4, const float* rows0, int64_t row_stride,
                                               int row_group, int64_t p0, int64_t L) {
  for (int i0 = threadIdx.x; i0 < n4; i0 += kThreads * PU) {
    float4 acc[PU];
#pragma unroll
    for (int u = 0; u < PU; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r0 = 0; r0 < row_group; r0 += RU) {
      float4 x[RU][PU];
#pragma unroll
      for (int ru = 0; ru < RU; ++ru) {
        const float* row = rows0 + (int64_t)(r0 + ru) * row_stride;
#pragma unroll
        for (int u = 0; u < PU; ++u) {
          const int i = i0 + u * kThreads;
          const int64_t pos = p0 + 4 * (int64_t)i;
          x[ru][u] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (r0 + ru < row_group && i < n4) {
            if (pos >= 0 && pos + 4 <= L) {
              x[ru][u] = *reinterpret_cast<const float4*>(row + pos);
            } else {
              if (pos + 0 >= 0 && pos + 0 < L) x[ru][u].x = row[pos + 0];
              if (pos + 1 >= 0 && pos + 1 < L) x[ru][u].y = row[pos + 1];
              if (pos + 2 >= 0 && pos + 2 < L) x[ru][u].z = row[pos + 2];
              if (pos + 3 >= 0 && pos + 3 < L) x[ru][u].w = row[pos + 3];
            }
          }
        }
      }
#pragma unroll
      for (int ru = 0; ru < RU; ++ru) {
        if (r0 + ru >= row_group) break;
#pragma unroll
        for (int u = 0; u < PU; ++u) {
          acc[u].x += x[ru][u].x;
          acc[u].y += x[ru][u].y;
          acc[u].z += x[ru][u].z;
          acc[u].w += x[ru][u].w;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < PU; ++u)
      if (i0 + u * kThreads < n4) st4[i0 + u * kThreads] = acc[u];
  }
}

template <int CS>
__global__ void __launch_bounds__(kThreads, 1) select_kernel(const SelArgs a) {
  pdl_wait();
  __shared__ SelShared sh;
  extern __shared__ __align__(16) float dyn[];
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = (int)cluster.block_rank();
  const int o = blockIdx.y;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool varlen = a.cu != nullptr;

  int64_t start = 0, len = a.n;
  bool bad = false;
  if (varlen) {
    start = a.cu[b];
    len = (int64_t)a.cu[b + 1] - start;
    bad = (start < 0 || len < a.w || start + len > a.n);  // a.n: packed total of the batch
    // a sequence longer than the max_seqlen the launch was sized for
    if (!bad && a.smem_vals && sel_segment(len - a.w, CS) > a.seg_cap) bad = true;
  }
  const int64_t orow = varlen ? ((int64_t)b * a.out_rows + o) : o;
  int32_t* out = a.idx + orow * (varlen ? a.k : a.idx_row_stride);
  const int64_t kout = varlen ? a.k : (a.k < a.n ? a.k : a.n);  // entries written in this row

  if (bad) {  // malformed sequence: report, pad, and stop (uniform per cluster)
    if (crank == 0 && threadIdx.x == 0) {
      set_dev_err(a.err, KVC_DEV_ERR_SEQLENS);
      if (a.counts && o == 0) a.counts[b] = 0;
    }
    for (int64_t t = (int64_t)crank * kThreads + threadIdx.x; t < kout; t += (int64_t)CS * kThreads)
      out[t] = -1;
    return;
  }
  const int64_t m = a.k < len ? a.k : len;  // positions kept in this sequence
  if (varlen && a.counts && o == 0 && crank == 0 && threadIdx.x == 0) a.counts[b] = (int32_t)m;
  // padding of short sequences (varlen rows have k entries)
  for (int64_t t = m + (int64_t)crank * kThreads + threadIdx.x; t < kout; t += (int64_t)CS * kThreads)
    out[t] = -1;

  const int64_t L = len - a.w;
  const int64_t kk = a.k - a.w;
  if (a.k >= len) {  // keep everything
    for (int64_t t = (int64_t)crank * kThreads + threadIdx.x; t < len; t += (int64_t)CS * kThreads)
      out[t] = (int32_t)t;
  } else {
    for (int64_t t = (int64_t)crank * kThreads + threadIdx.x; t < a.w; t += (int64_t)CS * kThreads)
      out[kk + t] = (int32_t)(L + t);
  }
  const bool need_rank = (a.k < len) && kk > 0;
  if (!need_rank && a.vals_g == nullptr) return;  // nothing to rank, nothing to report

  // ---- segment of this CTA: row sums (+halo), then pooled values -------------
  const int64_t seg = sel_segment(L, CS);
  const int64_t s0 = (int64_t)crank * seg < L ? (int64_t)crank * seg : L;
  const int64_t s1 = s0 + seg < L ? s0 + seg : L;
  const int nseg = (int)(s1 - s0);
  const int half = a.pool / 2;
  const float pool_div = (float)a.pool;
  const float* rows0 = a.scores + (int64_t)o * a.row_group * a.row_stride + start;
  float* gvals = a.vals_g ? a.vals_g + (int64_t)o * a.vals_stride + (a.vals_packed ? start : 0) : nullptr;
  // pooled values of the segment, indexed 0..nseg-1 (shared or global memory)
  float* v = a.smem_vals ? dyn + a.v_off : gvals + s0;

  for (int i = threadIdx.x; i < kBins; i += kThreads) sh.rx.hist[0][i] = 0;
  if (threadIdx.x == 0) sh.cand_n = 0;

  if (a.smem_vals) {
    // row sums R over [s0 - hs, s0 + nseg4 + hs + 4) into the stage, zero
    // outside [0, L)
    const int hs = stage_halo(half);
    const int nseg4 = (nseg + 3) & ~3;
    float* stage = dyn;
    const int64_t p0 = s0 - hs;
    const int span = nseg4 + 2 * hs + 4;
    const bool vec_in = ((reinterpret_cast<uintptr_t>(rows0) & 15) == 0) && (a.row_stride & 3) == 0 && (p0 & 3) == 0;
    if (vec_in) {
      float4* st4 = reinterpret_cast<float4*>(stage);
      const int n4 = span / 4;
      if (a.row_group >= 8)
        stage_row_sums<8, 1>(st4, n4, rows0, a.row_stride, a.row_group, p0, L);
      else if (a.row_group >= 4)
        stage_row_sums<4, 2>(st4, n4, rows0, a.row_stride, a.row_group, p0, L);
      else if (a.row_group >= 2)
        stage_row_sums<2, 2>(st4, n4, rows0, a.row_stride, a.row_group, p0, L);
      else
        stage_row_sums<1, 4>(st4, n4, rows0, a.row_stride, a.row_group, p0, L);
    } else {
      // unaligned rows: coalesced 4-byte loads, eight positions per thread in flight
      constexpr int kU = 8;
      for (int t0 = threadIdx.x; t0 < span; t0 += kThreads * kU) {
        float acc[kU];
        bool ok[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int64_t pos = p0 + t0 + u * kThreads;
          ok[u] = t0 + u * kThreads < span && pos >= 0 && pos < L;
          acc[u] = 0.f;
        }
        for (int r = 0; r < a.row_group; ++r) {
          const float* row = rows0 + (int64_t)r * a.row_stride + p0 + t0;
#pragma unroll
          for (int u = 0; u < kU; ++u)
            if (ok[u]) acc[u] += row[u * kThreads];
        }
#pragma unroll
        for (int u = 0; u < kU; ++u)
          if (t0 + u * kThreads < span) stage[t0 + u * kThreads] = acc[u];
      }
    }
    __syncthreads();
  } else {
    // long rows: pooled values go straight to global memory (L2-resident)
    for (int t = threadIdx.x; t < nseg; t += kThreads) {
      float sum = 0.f;
      for (int q = -half; q <= half; ++q) {
        const int64_t pos = s0 + t + q;
        if (pos < 0 || pos >= L) continue;
        float rs = 0.f;
        for (int r = 0; r < a.row_group; ++r) rs += rows0[(int64_t)r * a.row_stride + pos];
        sum += rs;
      }
      v[t] = sum;  // ranked as the pooled sum (see the shared-memory path)
    }
    __syncthreads();
  }
  // global-memory mode keeps the pooled sums in the caller's buffer while
  // ranking; it holds the averages once this CTA no longer reads them
  auto finish_gvals = [&]() {
    if (!a.smem_vals && gvals && a.pool > 1) {
      __syncthreads();
      for (int t = threadIdx.x; t < nseg; t += kThreads) v[t] = v[t] / pool_div;
    }
  };
  const PooledKeys pk{a.smem_vals ? reinterpret_cast<const uint32_t*>(v) : nullptr, v};
  const int hs = stage_halo(half);
  const float* stage = dyn;
  // Pooled sum of position t from the staged row sums (ascending order, the
  // same as the pooling pass below).
  auto pooled_at = [&](int t) {
    float sum = 0.f;
    for (int q = -half; q <= half; ++q) sum += stage[t + hs + q];
    return sum;
  };
  // Shared-memory mode: the pooling pass.  v holds order keys of the sums p*S
  // (ranking uses the sum: the average differs by the constant factor 1/p, a
  // monotone map, so the order -- ties to the lower position -- is the same;
  // the average itself is only formed for the optional pooled output).  Each
  // thread forms four consecutive outputs from 16-byte shared-memory loads
  // (lanes 128 positions apart: no bank conflicts, and neighbouring -- similar
  // -- values rarely hit one histogram bin in the same instruction); `bin`
  // maps keys to histogram bins, or is null.
  auto pool_pass = [&](auto&& bin, bool with_hist) {
    const float4* st4 = reinterpret_cast<const float4*>(stage);
    uint4* v4 = reinterpret_cast<uint4*>(v);
    const int nv = ((nseg + 3) & ~3) / 4;
    for (int i = spread_index(warp, lane); i < nv; i += kThreads) {
      float sums[4];
      if (hs == 0) {
        const float4 x = st4[i];
        sums[0] = x.x;
        sums[1] = x.y;
        sums[2] = x.z;
        sums[3] = x.w;
      } else if (hs == 4) {
        const float4 x0 = st4[i], x1 = st4[i + 1], x2 = st4[i + 2];
        const float win[12] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w, x2.x, x2.y, x2.z, x2.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float sum = 0.f;
#pragma unroll
          for (int q = 0; q <= 8; ++q)
            if (q >= 4 - half && q <= 4 + half) sum += win[u + q];
          sums[u] = sum;
        }
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) sums[u] = pooled_at(4 * i + u);
      }
      uint32_t key[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) key[u] = order_key(sums[u]);
      v4[i] = make_uint4(key[0], key[1], key[2], key[3]);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const bool in = 4 * i + u < nseg;
        if (in && gvals) gvals[s0 + 4 * i + u] = (a.pool == 1) ? sums[u] : sums[u] / pool_div;
        if (with_hist) hist_add(sh.rx.hist[0], bin(key[u]), in);
      }
    }
  };
  if (!need_rank) {
    if (a.smem_vals) pool_pass([](uint32_t) { return 0u; }, false);
    finish_gvals();
    return;
  }

  // ---- 1. sample -> key window --------------------------------------------------
  // every CTA samples evenly spaced pooled values of its segment; the sample
  // counts per rank follow from the segment lengths, so each CTA knows them
  constexpr int kPer = kSampleTotal / CS;
  if (warp == 0) {
    uint32_t c = 0;
    if (lane < CS) {
      const int64_t r0 = (int64_t)lane * seg < L ? (int64_t)lane * seg : L;
      const int64_t nr = L - r0 < seg ? L - r0 : seg;
      c = (uint32_t)(nr < kPer ? nr : kPer);
    }
    const uint32_t ex = warp_excl_scan(c);
    if (lane <= CS) sh.soff[lane] = ex;
  }
  {
    const int nsc = nseg < kPer ? nseg : kPer;
    if (threadIdx.x < nsc) {
      const int t = (int)(((2 * (int64_t)threadIdx.x + 1) * nseg) / (2 * nsc));
      sh.sample[threadIdx.x] = a.smem_vals ? order_key(pooled_at(t)) : order_key(v[t]);
    }
  }
  cluster.sync();
  const uint32_t ns = sh.soff[CS];
  if (threadIdx.x < ns) {
    int r = 0;
#pragma unroll
    for (int q = 1; q < CS; ++q) r += sh.soff[q] <= threadIdx.x;
    sh.sall[threadIdx.x] = cluster.map_shared_rank(&sh, r)->sample[threadIdx.x - sh.soff[r]];
  }
  __syncthreads();
  {
    // rank by counting (equal keys: lower slot first), eight threads per sample
    const uint32_t i = threadIdx.x >> 3, part = threadIdx.x & 7;
    const uint32_t mine = i < ns ? sh.sall[i] : 0u;
    uint32_t c = 0;
    if (i < ns) {
#pragma unroll 4
      for (uint32_t j = part; j < ns; j += 8) {
        const uint32_t x = sh.sall[j];
        c += (x > mine) || (x == mine && j < i);
      }
    }
    c += __shfl_xor_sync(0xffffffffu, c, 1);
    c += __shfl_xor_sync(0xffffffffu, c, 2);
    c += __shfl_xor_sync(0xffffffffu, c, 4);
    if (i < ns && part == 0) sh.ssort[c] = mine;
  }
  __syncthreads();
  // the kk-th largest key sits near sample index ns*kk/L; the window spans
  // `margin` sample places to either side
  const int tr = min((int)ns - 1, (int)((float)ns * ((float)kk / (float)L)));
  const int margin = 4 + (int)ns / 16;
  const uint32_t hi_key = tr - margin >= 0 ? sh.ssort[tr - margin] : 0xFFFFFFFFu;
  const uint32_t lo_key = tr + margin < (int)ns ? sh.ssort[tr + margin] : 0u;
  const uint32_t wdt = hi_key - lo_key;
  const int wsh = wdt < (uint32_t)kWin ? 0 : 32 - __clz(wdt / (uint32_t)kWin);  // (wdt >> wsh) < kWin
  auto wbin = [&](uint32_t key) -> uint32_t {
    if (key < lo_key) return 0u;
    const uint32_t d = (key - lo_key) >> wsh;
    return d >= (uint32_t)kWin ? (uint32_t)(kWinBins - 1) : d + 1u;
  };

  // ---- 2. windowed histogram (with the pooling pass), summed over the cluster --
  if (a.smem_vals) {
    pool_pass(wbin, true);
  } else {
    for (int t0 = 0; t0 < nseg; t0 += kThreads) {
      const int t = t0 + spread_index(warp, lane);
      if (t < nseg) hist_add(sh.rx.hist[0], wbin(pk.at(t)), true);
    }
  }
  cluster.sync();
  cluster_find_bucket<CS>(cluster, sh.rx, 0, kWinBins, (uint32_t)kk);
  const uint32_t b1 = sh.rx.found_bucket & (kWinBins - 1);
  const uint32_t nc = (uint32_t)sh.rx.tot[b1];
  const bool listed = b1 != 0u && b1 != (uint32_t)(kWinBins - 1) && nc <= (uint32_t)kCandMax;  // uniform

  // compaction layout: warp w owns positions [w*sub, (w+1)*sub) of the
  // segment, four consecutive positions per lane and step
  const int sub = (nseg + kThreads * 4 - 1) / (kThreads * 4) * 128;
  const int w0 = min(nseg, warp * sub), w1 = min(nseg, w0 + sub);

  uint32_t T, need_eq;              // threshold key; how many keys == T are taken
  uint32_t g_prev = 0, e_prev = 0;  // keys > T / == T in the lower ranks
  if (listed) {
    // ---- 3. candidates (keys of bin b1) with positions, rank by rank ----------
    if (warp == 0) {
      const uint32_t c = lane < CS ? (uint32_t)cluster.map_shared_rank(&sh.rx.hist[0][0], lane)[b1] : 0u;
      const uint32_t ex = warp_excl_scan(c);
      if (lane <= CS) sh.cand_off[lane] = ex;
    }
    __syncthreads();
    const uint32_t off = sh.cand_off[crank];
    uint32_t above_w = 0;  // keys of this warp's range in bins above b1
    for (int p = w0 + 4 * lane; p - 4 * lane < w1; p += 128) {
      uint32_t key[4];
      pk.four(p, w1, key);
      uint32_t nmine = 0;
      bool is[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t bin = wbin(key[q]);
        const bool in = p + q < w1;
        above_w += in && bin > b1;
        is[q] = in && bin == b1;
        nmine += is[q];
      }
      if (__any_sync(0xffffffffu, nmine != 0)) {  // candidates are rare: most steps skip this
        const uint32_t ex = warp_excl_scan(nmine);
        const uint32_t tot = __shfl_sync(0xffffffffu, ex + nmine, 31);
        uint32_t base = 0;
        if (lane == 0) base = atomicAdd(&sh.cand_n, tot);
        base = __shfl_sync(0xffffffffu, base, 0) + off + ex;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (is[q]) sh.cand[base++] = make_uint2(key[q], (uint32_t)(p + q));
      }
    }
    above_w = warp_sum(above_w);
    if (lane == 0) {
      sh.warp_gt[warp] = above_w;
      sh.warp_eq[warp] = 0;
    }
    __syncthreads();
    if (warp == 0) {
      const uint32_t t = warp_sum(sh.warp_gt[lane]);
      if (lane == 0) sh.above = t;
    }
    cluster.sync();  // every rank's candidates and `above` are published
    // gather the other ranks' candidates
    const uint32_t own_n = sh.cand_off[crank + 1] - off;
    for (uint32_t i = threadIdx.x; i < nc; i += kThreads) {
      if (i >= off && i < off + own_n) continue;
      int r = 0;
#pragma unroll
      for (int q = 1; q < CS; ++q) r += sh.cand_off[q] <= i;
      sh.cand[i] = cluster.map_shared_rank(&sh.cand[0], r)[i];
    }
    uint32_t above_prev = 0;
    if (warp == 0) above_prev = warp_sum(lane < crank ? cluster.map_shared_rank(&sh, lane)->above : 0u);
    __syncthreads();
    // the want-th largest candidate.  Every candidate lies in bin b1, i.e.
    // its key is base + off with off < 2^wsh.  Up to two 11-bit histogram
    // levels over off narrow a long list down to the keys that agree above
    // the last `rest` bits; those are ranked by counting (four threads per
    // key).  Lists alternate between hist[0] and tot (free by now: no CTA
    // reads this CTA's histograms after the last cluster barrier).
    {
      uint32_t want = sh.rx.found_rem;
      const uint32_t base = lo_key + ((b1 - 1u) << wsh);
      uint32_t* lst = reinterpret_cast<uint32_t*>(sh.rx.hist[0]);
      uint32_t* nxt = reinterpret_cast<uint32_t*>(sh.rx.tot);
      for (uint32_t i = threadIdx.x; i < nc; i += kThreads) lst[i] = sh.cand[i].x - base;
      if (threadIdx.x == 0) sh.cand_n = 0;
      __syncthreads();
      uint32_t n = nc;
      int rest = wsh;
      for (int level = 0; level < 2 && n > 64 && rest > 0; ++level) {
        const int sb = rest < 11 ? rest : 11;
        const int shf = rest - sb;
        const uint32_t mask = (1u << sb) - 1u;
        for (int i = threadIdx.x; i < kBins; i += kThreads) sh.rx.hist[1][i] = 0;
        __syncthreads();
        for (uint32_t i = threadIdx.x; i < n; i += kThreads) atomicAdd(&sh.rx.hist[1][(lst[i] >> shf) & mask], 1);
        __syncthreads();
        scan_find(sh.rx, sh.rx.hist[1], kBins, want);
        const uint32_t sbin = sh.rx.found_bucket & mask;
        want = sh.rx.found_rem;
        for (uint32_t i = threadIdx.x; i < n; i += kThreads) {
          const uint32_t x = lst[i];
          if (((x >> shf) & mask) == sbin) nxt[atomicAdd(&sh.cand_n, 1u)] = x;
        }
        __syncthreads();
        n = sh.cand_n;
        __syncthreads();
        if (threadIdx.x == 0) sh.cand_n = 0;
        uint32_t* t = lst;
        lst = nxt;
        nxt = t;
        rest = shf;
      }
      if (rest == 0) {  // the survivors are all equal
        if (threadIdx.x == 0) {
          sh.T = base + lst[0];
          sh.need_eq = want;
        }
      } else {
        for (uint32_t i0 = 0; i0 < n; i0 += kThreads / 4) {
          const uint32_t i = i0 + (threadIdx.x >> 2), part = threadIdx.x & 3;
          const uint32_t mine = i < n ? lst[i] : 0u;
          uint32_t gt = 0, eq = 0;
          if (i < n) {
#pragma unroll 4
            for (uint32_t j = part; j < n; j += 4) {
              const uint32_t x = lst[j];
              gt += x > mine;
              eq += x == mine;
            }
          }
          gt += __shfl_xor_sync(0xffffffffu, gt, 1);
          gt += __shfl_xor_sync(0xffffffffu, gt, 2);
          eq += __shfl_xor_sync(0xffffffffu, eq, 1);
          eq += __shfl_xor_sync(0xffffffffu, eq, 2);
          if (i < n && part == 0 && gt < want && want <= gt + eq) {
            sh.T = base + mine;
            sh.need_eq = want - gt;
          }
        }
      }
    }
    __syncthreads();
    T = sh.T;
    need_eq = sh.need_eq;
    // this CTA's candidates per compaction warp; the lower ranks' candidates
    for (uint32_t i = off + threadIdx.x; i < off + own_n; i += kThreads) {
      const uint2 c = sh.cand[i];
      const int w = sub > 0 ? (int)c.y / sub : 0;
      if (c.x > T) atomicAdd(&sh.warp_gt[w], 1u);
      if (c.x == T) atomicAdd(&sh.warp_eq[w], 1u);
    }
    uint32_t gt = threadIdx.x == 0 ? above_prev : 0u, eq = 0;
    for (uint32_t i = threadIdx.x; i < off; i += kThreads) {
      const uint32_t x = sh.cand[i].x;
      gt += x > T;
      eq += x == T;
    }
    block_sum2(gt, eq, sh.red);  // (also completes the per-warp atomics)
    g_prev = gt;
    e_prev = eq;
  } else {
    // ---- the window missed, or heavy ties: plain radix select, cluster-wide ----
    // (hist[1] and hist[0] alternate: a CTA rewrites a histogram only after the
    // cluster barrier that follows every rank's last read of it)
    uint32_t want = (uint32_t)kk;
    for (int i = threadIdx.x; i < kBins; i += kThreads) sh.rx.hist[1][i] = 0;
    __syncthreads();
    for (int t0 = 0; t0 < nseg; t0 += kThreads) {
      const int t = t0 + spread_index(warp, lane);
      if (t < nseg) hist_add(sh.rx.hist[1], pk.at(t) >> 21, true);
    }
    cluster.sync();
    cluster_find_bucket<CS>(cluster, sh.rx, 1, kBins, want);
    const uint32_t r1 = sh.rx.found_bucket & (kBins - 1);
    want = sh.rx.found_rem;
    for (int i = threadIdx.x; i < kBins; i += kThreads) sh.rx.hist[0][i] = 0;
    __syncthreads();
    for (int t0 = 0; t0 < nseg; t0 += kThreads) {
      const int t = t0 + spread_index(warp, lane);
      const uint32_t key = t < nseg ? pk.at(t) : 0u;
      hist_add(sh.rx.hist[0], (key >> 10) & 2047u, t < nseg && (key >> 21) == r1);
    }
    cluster.sync();
    cluster_find_bucket<CS>(cluster, sh.rx, 0, kBins, want);
    const uint32_t pre2 = (r1 << 11) | (sh.rx.found_bucket & (kBins - 1));
    want = sh.rx.found_rem;
    for (int i = threadIdx.x; i < kBins; i += kThreads) sh.rx.hist[1][i] = 0;
    __syncthreads();
    for (int t0 = 0; t0 < nseg; t0 += kThreads) {
      const int t = t0 + spread_index(warp, lane);
      const uint32_t key = t < nseg ? pk.at(t) : 0u;
      hist_add(sh.rx.hist[1], key & 1023u, t < nseg && (key >> 10) == pre2);
    }
    cluster.sync();
    cluster_find_bucket<CS>(cluster, sh.rx, 1, 1024, want);
    T = (pre2 << 10) | (sh.rx.found_bucket & 1023u);
    need_eq = sh.rx.found_rem;
    // per-warp counts, then the per-CTA totals through the cluster
    {
      uint32_t gt = 0, eq = 0;
      for (int p = w0 + 4 * lane; p < w1; p += 128) {
        uint32_t key[4];
        pk.four(p, w1, key);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          gt += p + q < w1 && key[q] > T;
          eq += p + q < w1 && key[q] == T;
        }
      }
      gt = warp_sum(gt);
      eq = warp_sum(eq);
      if (lane == 0) {
        sh.warp_gt[warp] = gt;
        sh.warp_eq[warp] = eq;
      }
    }
    __syncthreads();
    if (warp == 0) {
      const uint32_t tg = warp_sum(sh.warp_gt[lane]), te = warp_sum(sh.warp_eq[lane]);
      if (lane == 0) {
        sh.cnt_gt = tg;
        sh.cnt_eq = te;
      }
    }
    cluster.sync();
    if (warp == 0) {
      uint32_t g = 0, e = 0;
      if (lane < crank) {
        const SelShared* r = cluster.map_shared_rank(&sh, lane);
        g = r->cnt_gt;
        e = r->cnt_eq;
      }
      g = warp_sum(g);
      e = warp_sum(e);
      if (lane == 0) {
        sh.g_prev = g;
        sh.e_prev = e;
      }
    }
    __syncthreads();
    g_prev = sh.g_prev;
    e_prev = sh.e_prev;
  }
  cluster_arrive();  // no reads of other CTAs' shared memory from here on

  // ---- order-preserving compaction ---------------------------------------------
  {
    uint32_t run_g = g_prev + warp_sum(lane < warp ? sh.warp_gt[lane] : 0u);
    uint32_t run_e = e_prev + warp_sum(lane < warp ? sh.warp_eq[lane] : 0u);
    const uint32_t kk32 = (uint32_t)kk;  // output slots of the ranked part (bounds guard)
    for (int p = w0 + 4 * lane; p - 4 * lane < w1; p += 128) {
      uint32_t key[4];
      pk.four(p, w1, key);
      uint32_t ng = 0, ne = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        ng += p + q < w1 && key[q] > T;
        ne += p + q < w1 && key[q] == T;
      }
      const uint32_t packed = warp_excl_scan(ng | (ne << 16));
      uint32_t gb = run_g + (packed & 0xffffu);  // keys > T before this lane's first
      uint32_t eb = run_e + (packed >> 16);      // keys == T before it
      const uint32_t tot = __shfl_sync(0xffffffffu, packed + (ng | (ne << 16)), 31);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool in = p + q < w1;
        const bool g = in && key[q] > T, e = in && key[q] == T;
        const uint32_t slot = gb + min(eb, need_eq);
        if ((g || (e && eb < need_eq)) && slot < kk32) out[slot] = (int32_t)(s0 + p + q);
        gb += g;
        eb += e;
      }
      run_g += tot & 0xffffu;
      run_e += tot >> 16;
    }
  }
  finish_gvals();
  cluster_wait();  // other CTAs' reads of this CTA's shared memory are over
}

// --------------------------------------------------------------------------
// statistics
// --------------------------------------------------------------------------
struct StatArgs {
  const float* scores;
  int64_t row_stride;
  int64_t n;
  float inv_mass;
  float* out;
};

struct StatShared {
  RadixShared rx;
  double red[kWarps];
  double part[3];  // this CTA's partial sums, read by the cluster
};

// Block-wide sum of a double (all threads get the result).
__device__ double block_sum(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double s = 0.0;
  for (int i = 0; i < kWarps; ++i) s += red[i];
  return s;
}

__global__ void __cluster_dims__(kCS, 1, 1) __launch_bounds__(kThreads, 1)
stats_kernel(const StatArgs a) {
  pdl_wait();
  pdl_trigger();
  __shared__ StatShared sh;
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = (int)cluster.block_rank();
  const int r = blockIdx.y;
  const float* row = a.scores + (int64_t)r * a.row_stride;
  const int64_t seg = (a.n + kCS - 1) / kCS;
  const int64_t s0 = (int64_t)crank * seg < a.n ? (int64_t)crank * seg : a.n;
  const int64_t s1 = s0 + seg < a.n ? s0 + seg : a.n;
  const int64_t m = (a.n + 99) / 100;

  for (int i = threadIdx.x; i < kBins; i += kThreads) sh.rx.hist[0][i] = 0;
  __syncthreads();
  float sum = 0.f, ent = 0.f;
  for (int64_t j = s0 + threadIdx.x; j < s1; j += kThreads) {
    const float v = row[j] * a.inv_mass;
    sum += v;
    if (v > 0.f) ent -= v * logf(v);
    atomicAdd(&sh.rx.hist[0][order_key(v) >> 21], 1);
  }
  double bs = block_sum(sum, sh.red);
  double be = block_sum(ent, sh.red);
  if (threadIdx.x == 0) {
    sh.part[0] = bs;
    sh.part[1] = be;
  }
  cluster.sync();
  double tsum = 0.0, tent = 0.0;
  for (int c = 0; c < kCS; ++c) {
    StatShared* rs = cluster.map_shared_rank(&sh, c);
    tsum += rs->part[0];
    tent += rs->part[1];
  }
  const float mean = (float)(tsum / (double)a.n);

  cluster_find_bucket<kCS>(cluster, sh.rx, 0, kBins, (uint32_t)m);
  const uint32_t b1 = sh.rx.found_bucket;
  uint32_t want = sh.rx.found_rem;
  for (int i = threadIdx.x; i < kBins; i += kThreads) sh.rx.hist[1][i] = 0;
  __syncthreads();
  for (int64_t j = s0 + threadIdx.x; j < s1; j += kThreads) {
    const uint32_t key = order_key(row[j] * a.inv_mass);
    if ((key >> 21) == b1) atomicAdd(&sh.rx.hist[1][(key >> 10) & 2047u], 1);
  }
  cluster.sync();
  cluster_find_bucket<kCS>(cluster, sh.rx, 1, kBins, want);
  const uint32_t pre2 = (b1 << 11) | sh.rx.found_bucket;
  want = sh.rx.found_rem;
  for (int i = threadIdx.x; i < kBins; i += kThreads) sh.rx.hist[0][i] = 0;
  __syncthreads();
  for (int64_t j = s0 + threadIdx.x; j < s1; j += kThreads) {
    const uint32_t key = order_key(row[j] * a.inv_mass);
    if ((key >> 10) == pre2) atomicAdd(&sh.rx.hist[0][key & 1023u], 1);
  }
  cluster.sync();
  cluster_find_bucket<kCS>(cluster, sh.rx, 0, 1024, want);
  const uint32_t T = (pre2 << 10) | sh.rx.found_bucket;
  const uint32_t need_eq = sh.rx.found_rem;

  float top = 0.f, var = 0.f;
  for (int64_t j = s0 + threadIdx.x; j < s1; j += kThreads) {
    const float v = row[j] * a.inv_mass;
    if (order_key(v) > T) top += v;
    const float dv = v - mean;
    var += dv * dv;
  }
  double bt = block_sum(top, sh.red);
  double bv = block_sum(var, sh.red);
  // the part[] slots are re-used: every CTA finished reading them above
  // (cluster barriers inside cluster_find_bucket separate the two phases)
  cluster.sync();
  if (threadIdx.x == 0) {
    sh.part[0] = bt;
    sh.part[2] = bv;
  }
  cluster.sync();
  if (crank == 0 && threadIdx.x == 0) {
    double ttop = 0.0, tvar = 0.0;
    for (int c = 0; c < kCS; ++c) {
      StatShared* rs = cluster.map_shared_rank(&sh, c);
      ttop += rs->part[0];
      tvar += rs->part[2];
    }
    ttop += (double)need_eq * (double)key_value(T);
    a.out[3 * r + 0] = (float)tent;
    a.out[3 * r + 1] = (float)ttop;
    a.out[3 * r + 2] = (float)(tvar / (double)a.n);
  }
  cluster.sync();
}

constexpr size_t kSelDynMax = 184 * 1024;  // dynamic smem of the selection kernel

// pooled segment (and its staged row sums) of `seg` positions fit in shared memory
bool sel_fits_smem(int64_t seg, int half) {
  return (sel_v_words(seg) + sel_stage_words(seg, half)) * sizeof(float) <= kSelDynMax;
}

// Whether this device can place a 16-CTA selection cluster (looked up once per
// context; the kernel attributes are set on the way).
bool wide_clusters_available() {
  static ContextCache cache;
  static bool ok[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  const kvc_status s = once_per_context(cache, [dev] {
    ok[dev] = false;
    KVC_CUDA_TRY(cudaFuncSetAttribute(select_kernel<kCS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kSelDynMax));
    KVC_CUDA_TRY(cudaFuncSetAttribute(select_kernel<kCSWide>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kSelDynMax));
    if (cudaFuncSetAttribute(select_kernel<kCSWide>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
        cudaSuccess) {
      cudaGetLastError();
      return KVC_OK;
    }
    Launch l(dim3(kCSWide, 1, 1), dim3(kThreads), kSelDynMax, nullptr);
    l.cluster_x(kCSWide);
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, select_kernel<kCSWide>, &l.cfg) == cudaSuccess)
      ok[dev] = clusters > 0;
    else
      cudaGetLastError();
    return KVC_OK;
  });
  return s == KVC_OK && ok[dev];
}

// CTAs per ranking row: a lone long row (the all-head TSP row of a long
// sequence) is spread over a 16-CTA cluster when the device can place one --
// half the keys per CTA, and it runs alone -- every other launch uses 8.
int select_cluster_size(int rows_total, int64_t L) {
  return (rows_total == 1 && L >= kWideMinKeys && wide_clusters_available()) ? kCSWide : kCS;
}

// Launch: cs-CTA clusters, one per (sequence, output row).
kvc_status launch_select(SelArgs a, int out_rows, int batch, int cs, cudaStream_t st) {
  a.v_off = a.smem_vals ? (int)sel_stage_words(a.seg_cap, a.pool / 2) : 0;
  wide_clusters_available();  // sets the kernel attributes once per context
  Launch l(dim3(cs, out_rows, batch), dim3(kThreads), kSelDynMax, st);
  l.cluster_x(cs);
  if (cs == kCSWide)
    KVC_CUDA_TRY(l.run(select_kernel<kCSWide>, a));
  else
    KVC_CUDA_TRY(l.run(select_kernel<kCS>, a));
  count_launch();
  return KVC_OK;
}

kvc_status check_select_common(const float* scores, int32_t rows, int64_t row_stride,
                               int32_t row_group, int32_t w, int32_t pool, int64_t k,
                               const int32_t* idx) {
  KVC_CHECK_ARG(scores && idx, "scores and idx must be non-NULL");
  KVC_CHECK_ARG(rows >= 1 && row_group >= 1 && rows % row_group == 0,
                "rows must be a positive multiple of row_group");
  KVC_CHECK_ARG(rows / row_group <= 65535, "too many output rows");
  KVC_CHECK_ARG(w >= 1, "window must be >= 1");
  KVC_CHECK_ARG(pool >= 1 && (pool & 1) && pool / 2 <= kMaxHalf, "pool_kernel must be odd, 1..65");
  KVC_CHECK_ARG(k >= w && k < (int64_t(1) << 31), "k must be >= window and < 2^31");
  KVC_CHECK_ARG(row_stride >= 0, "row_stride must be >= 0");
  return KVC_OK;
}

}  // namespace
}  // namespace kvc

using namespace kvc;

extern "C" kvc_status kvc_select_workspace_size(int32_t out_rows, int32_t batch, int64_t total_tokens,
                                                size_t* bytes) {
  clear_error();
  KVC_CHECK_ARG(bytes != nullptr, "bytes must be non-NULL");
  KVC_CHECK_ARG(out_rows >= 1 && batch >= 1 && total_tokens >= 0, "bad sizes");
  *bytes = round_up((size_t)out_rows * (size_t)total_tokens * sizeof(float), kWsAlign) + kWsAlign;
  return KVC_OK;
}

extern "C" kvc_status kvc_select_topk(const float* scores, int32_t rows, int64_t row_stride,
                                      int32_t row_group, int64_t n, int32_t window,
                                      int32_t pool_kernel, int64_t k, int32_t* idx,
                                      int64_t idx_row_stride, float* pooled, void* ws,
                                      size_t ws_bytes, void* stream) {
  clear_error();
  kvc_status s = check_select_common(scores, rows, row_stride, row_group, window, pool_kernel, k, idx);
  if (s != KVC_OK) return s;
  KVC_CHECK_ARG(n >= window && n < (int64_t(1) << 31), "need window <= n < 2^31");
  KVC_CHECK_ARG(row_stride >= n, "row_stride must be >= n");
  KVC_CHECK_ARG(idx_row_stride >= (k < n ? k : n), "idx_row_stride must be >= min(k, n)");
  const int out_rows = rows / row_group;
  SelArgs a{};
  a.scores = scores;
  a.row_stride = row_stride;
  a.row_group = row_group;
  a.cu = nullptr;
  a.n = n;
  a.w = window;
  a.pool = pool_kernel;
  a.k = k;
  a.idx = idx;
  a.idx_row_stride = idx_row_stride;
  a.counts = nullptr;
  a.out_rows = out_rows;
  a.err = nullptr;
  const int cs = select_cluster_size(out_rows, n - window);
  const int64_t seg = sel_segment(n - window, cs);
  a.smem_vals = sel_fits_smem(seg, pool_kernel / 2);
  a.seg_cap = seg;
  if (pooled) {
    a.vals_g = pooled;
    a.vals_stride = n - window;
    a.vals_packed = false;
  } else if (a.smem_vals) {
    a.vals_g = nullptr;
  } else {
    size_t need = 0;
    kvc_select_workspace_size(out_rows, 1, n, &need);
    if (!ws || ws_bytes < need || !aligned(ws, kWsAlign))
      return fail(KVC_ERR_WORKSPACE, "select workspace missing, too small or not 256-B aligned");
    a.vals_g = static_cast<float*>(ws);
    a.vals_stride = n;
    a.vals_packed = true;
  }
  return launch_select(a, out_rows, 1, cs, (cudaStream_t)stream);
}

extern "C" kvc_status kvc_select_topk_varlen(const float* scores, int32_t rows, int64_t row_stride,
                                             int32_t row_group, const int32_t* cu_seqlens,
                                             int32_t batch, int64_t total, int64_t max_seqlen,
                                             int32_t window, int32_t pool_kernel, int64_t k,
                                             int32_t* idx, int32_t* counts, void* ws,
                                             size_t ws_bytes, int32_t* dev_err, void* stream) {
  clear_error();
  kvc_status s = check_select_common(scores, rows, row_stride, row_group, window, pool_kernel, k, idx);
  if (s != KVC_OK) return s;
  KVC_CHECK_ARG(cu_seqlens != nullptr, "cu_seqlens must be non-NULL");
  KVC_CHECK_ARG(batch >= 1 && batch <= 65535, "batch out of range");
  KVC_CHECK_ARG(total >= 0 && total < (int64_t(1) << 31) && row_stride >= total, "bad total / row_stride");
  KVC_CHECK_ARG(max_seqlen >= 0, "max_seqlen must be >= 0");
  const int out_rows = rows / row_group;
  size_t need = 0;
  kvc_select_workspace_size(out_rows, batch, total, &need);
  const int64_t seg_max = sel_segment(std::max<int64_t>(max_seqlen, window) - window, kCS);
  if (!sel_fits_smem(seg_max, pool_kernel / 2) &&
      (!ws || ws_bytes < need || !aligned(ws, kWsAlign)))
    return fail(KVC_ERR_WORKSPACE, "select workspace missing, too small or not 256-B aligned");
  SelArgs a{};
  a.scores = scores;
  a.row_stride = row_stride;
  a.row_group = row_group;
  a.cu = cu_seqlens;
  a.n = total;
  a.w = window;
  a.pool = pool_kernel;
  a.k = k;
  a.idx = idx;
  a.idx_row_stride = k;
  a.counts = counts;
  a.vals_g = nullptr;
  a.vals_stride = total;
  a.vals_packed = true;
  a.out_rows = out_rows;
  a.err = dev_err;
  a.smem_vals = sel_fits_smem(seg_max, pool_kernel / 2);
  a.seg_cap = seg_max;
  if (!a.smem_vals) a.vals_g = static_cast<float*>(ws);
  return launch_select(a, out_rows, batch, kCS, (cudaStream_t)stream);
}

extern "C" kvc_status kvc_stats_workspace_size(int32_t rows, int64_t n, size_t* bytes) {
  clear_error();
  KVC_CHECK_ARG(bytes != nullptr && rows >= 1 && n >= 1, "bad arguments");
  *bytes = 0;
  return KVC_OK;
}

extern "C" kvc_status kvc_layer_stats(const float* scores, int32_t rows, int64_t row_stride, int64_t n,
                                      float mass_norm, float* out, void* ws, size_t ws_bytes,
                                      void* stream) {
  clear_error();
  (void)ws;
  (void)ws_bytes;
  KVC_CHECK_ARG(scores && out, "scores and out must be non-NULL");
  KVC_CHECK_ARG(rows >= 1 && rows <= 65535, "rows out of range");
  KVC_CHECK_ARG(n >= 1 && n < (int64_t(1) << 31) && row_stride >= n, "bad n / row_stride");
  KVC_CHECK_ARG(mass_norm > 0.f, "mass_norm must be > 0");
  StatArgs a{scores, row_stride, n, 1.0f / mass_norm, out};
  dim3 grid(kCS, rows, 1);
  const Launch l(grid, dim3(kThreads), 0, (cudaStream_t)stream);
  KVC_CUDA_TRY(l.run(stats_kernel, a));
  count_launch();
  return KVC_OK;
}
