// select.cu -- top-k with a forced window, and per-row attention statistics.
//
// FastKV (gist.science 2502.01068) section 2.A: the selected tokens go on
// together with the observation-window tokens; section 2.B: the TSP rate and
// the KV retention rate are independent budgets over the same scores.
// StructKV (gist.science 2604.06746) section 2.B: attention entropy, sparsity
// (here: mass of the top 1 % keys) and variance per layer.
//
// Design: one thread-block cluster of kCS CTAs per ranking row.  Each CTA owns
// a contiguous segment of the row.  The exact k-th largest key is found by a
// three-pass radix select (11 + 11 + 10 bits of an order-preserving uint32
// image of the fp32 score); each pass builds a shared-memory histogram per
// CTA and the cluster sums the kCS histograms through distributed shared
// memory.  The final compaction walks each segment in index order with a
// block-wide scan, so the output is ascending without a sort.  Ties at the
// threshold go to the lowest positions.
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
constexpr int kMaxHalf = 32;    // pool_kernel <= 65
constexpr int kBins = 2048;     // radix bins of the first two passes
constexpr int kPerTile = 4;     // elements per thread in the compaction tiles

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

// Sum of this CTA's local hist[lo+1 .. nbins) (all threads get it).
__device__ __forceinline__ uint32_t local_count_above(RadixShared& sh, int buf, int nbins, uint32_t lo) {
  uint32_t mine = 0;
  for (int b = threadIdx.x; b < nbins; b += kThreads)
    if ((uint32_t)b > lo) mine += (uint32_t)sh.hist[buf][b];
  uint32_t total;
  block_excl_scan(mine, sh.warp_tmp, &total);
  return total;
}

// After every CTA of the cluster filled hist[buf] (and a cluster barrier),
// sum the kCS histograms and find the bin that holds the want-th largest
// candidate: count(bins above) < want <= count(bins above) + tot[bin].
// Bins are visited from the top.  Returns through sh.found_*.
__device__ void cluster_find_bucket(cg::cluster_group& cluster, RadixShared& sh, int buf, int nbins,
                                    uint32_t want) {
  // 16-byte loads of every rank's histogram, all issued before the sum: one
  // round trip through distributed shared memory
  for (int v4 = threadIdx.x; v4 < nbins / 4; v4 += kThreads) {
    int4 part[kCS];
#pragma unroll
    for (int c = 0; c < kCS; ++c) part[c] = reinterpret_cast<const int4*>(cluster.map_shared_rank(&sh.hist[buf][0], c))[v4];
    int4 acc = part[0];
#pragma unroll
    for (int c = 1; c < kCS; ++c) {
      acc.x += part[c].x;
      acc.y += part[c].y;
      acc.z += part[c].z;
      acc.w += part[c].w;
    }
    reinterpret_cast<int4*>(sh.tot)[v4] = acc;
  }
  __syncthreads();
  // thread t owns the group of bins (kThreads-1-t): higher t = lower bins
  const int per = nbins / kThreads;  // 1 or 2
  const int grp = kThreads - 1 - threadIdx.x;
  uint32_t mine = 0;
  for (int q = 0; q < per; ++q) mine += sh.tot[grp * per + q];
  uint32_t total;
  uint32_t above = block_excl_scan(mine, sh.warp_tmp, &total);
  for (int q = per - 1; q >= 0; --q) {
    const int bin = grp * per + q;
    const uint32_t c = sh.tot[bin];
    if (above < want && want <= above + c) {
      sh.found_bucket = bin;
      sh.found_rem = want - above;
    }
    above += c;
  }
  __syncthreads();
}

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
  int out_rows;
  int32_t* err;
};

struct SelShared {
  RadixShared rx;
  uint32_t cnt_gt, cnt_eq;  // this CTA's counts for the output phase
};

// Histogram increment.  Contention is modest (a CTA's 16K keys spread over
// tens of first-pass bins; later passes only see the keys of one bucket), so
// plain shared-memory atomics beat warp-level match/aggregate here.
__device__ __forceinline__ void hist_add(int* hist, uint32_t bin, bool active) {
  if (active) atomicAdd(&hist[bin], 1);
}

// Dynamic shared memory of the selection kernel: the staged row sums of the
// segment plus halo, and the pooled values of the segment (smem mode).
__host__ __device__ inline size_t sel_dyn_smem(int64_t seg, int half, bool smem_vals) {
  return smem_vals ? (size_t)(2 * seg + 2 * half + 16) * sizeof(float) : 0;
}

__global__ void __cluster_dims__(kCS, 1, 1) __launch_bounds__(kThreads, 1)
select_kernel(const SelArgs a) {
  __shared__ SelShared sh;
  extern __shared__ float dyn[];
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = (int)cluster.block_rank();
  const int o = blockIdx.y;
  const int b = blockIdx.z;
  const bool varlen = a.cu != nullptr;

  int64_t start = 0, len = a.n;
  bool bad = false;
  if (varlen) {
    start = a.cu[b];
    len = (int64_t)a.cu[b + 1] - start;
    bad = (start < 0 || len < a.w);
    // a sequence longer than the max_seqlen the launch was sized for
    if (!bad && a.smem_vals && (len - a.w + kCS - 1) / kCS > a.seg_cap) bad = true;
  }
  const int64_t orow = varlen ? ((int64_t)b * a.out_rows + o) : o;
  int32_t* out = a.idx + orow * (varlen ? a.k : a.idx_row_stride);
  const int64_t kout = varlen ? a.k : (a.k < a.n ? a.k : a.n);  // entries written in this row

  if (bad) {  // malformed sequence: report, pad, and stop (uniform per cluster)
    if (crank == 0 && threadIdx.x == 0) {
      set_dev_err(a.err, KVC_DEV_ERR_SEQLENS);
      if (a.counts && o == 0) a.counts[b] = 0;
    }
    for (int64_t t = (int64_t)crank * kThreads + threadIdx.x; t < kout; t += (int64_t)kCS * kThreads)
      out[t] = -1;
    return;
  }
  const int64_t m = a.k < len ? a.k : len;  // positions kept in this sequence
  if (varlen && a.counts && o == 0 && crank == 0 && threadIdx.x == 0) a.counts[b] = (int32_t)m;
  // padding of short sequences (varlen rows have k entries)
  for (int64_t t = m + (int64_t)crank * kThreads + threadIdx.x; t < kout; t += (int64_t)kCS * kThreads)
    out[t] = -1;

  const int64_t L = len - a.w;
  const int64_t kk = a.k - a.w;
  if (a.k >= len) {  // keep everything
    for (int64_t t = (int64_t)crank * kThreads + threadIdx.x; t < len; t += (int64_t)kCS * kThreads)
      out[t] = (int32_t)t;
  } else {
    for (int64_t t = (int64_t)crank * kThreads + threadIdx.x; t < a.w; t += (int64_t)kCS * kThreads)
      out[kk + t] = (int32_t)(L + t);
  }
  const bool need_rank = (a.k < len) && kk > 0;
  if (!need_rank && a.vals_g == nullptr) return;  // nothing to rank, nothing to report

  // ---- segment of this CTA: row sums (+halo), then pooled values -------------
  const int64_t seg = (L + kCS - 1) / kCS;
  const int64_t s0 = (int64_t)crank * seg < L ? (int64_t)crank * seg : L;
  const int64_t s1 = s0 + seg < L ? s0 + seg : L;
  const int nseg = (int)(s1 - s0);
  const int half = a.pool / 2;
  const float pool_div = (float)a.pool;
  const float* rows0 = a.scores + (int64_t)o * a.row_group * a.row_stride + start;
  float* gvals = a.vals_g ? a.vals_g + (int64_t)o * a.vals_stride + (a.vals_packed ? start : 0) : nullptr;
  // pooled values of the segment, indexed 0..nseg-1 (shared or global memory)
  float* v = a.smem_vals ? dyn + ((nseg + 2 * half + 8 + 3) & ~3) : gvals + s0;  // 16-B aligned in smem

  for (int i = threadIdx.x; i < kBins; i += kThreads) sh.rx.hist[0][i] = 0;
  __syncthreads();

  constexpr int kU = 4;
  if (a.smem_vals) {
    float* stage = dyn;  // row sums over [s0 - half, s1 + half)
    const int span = nseg + 2 * half;
    for (int t0 = 0; t0 < span; t0 += kThreads * kU) {
      float acc[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) acc[u] = 0.f;
      for (int r = 0; r < a.row_group; ++r) {
        const float* row = rows0 + (int64_t)r * a.row_stride;
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int t = t0 + u * kThreads + threadIdx.x;
          const int64_t pos = s0 - half + t;
          if (t < span && pos >= 0 && pos < L) acc[u] += row[pos];
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int t = t0 + u * kThreads + threadIdx.x;
        if (t < span) stage[t] = acc[u];
      }
    }
    __syncthreads();
    // v[t] = sum of the p staged row sums around t.  Ranking uses this sum: the
    // average differs by the constant factor 1/p, a monotone map, so the order
    // (ties to the lower position) is the same; the average itself is only
    // formed for the optional pooled output.  Four consecutive outputs per
    // thread and round share one register window of 4 + 2*half staged values.
    const int span_w = 4 + 2 * half;
    for (int base = 0; base < nseg; base += 4 * kThreads) {
      const int t0 = base + 4 * threadIdx.x;
      float sums[4] = {0.f, 0.f, 0.f, 0.f};
      if (half <= 8) {
        float win[4 + 16];
#pragma unroll
        for (int q = 0; q < 4 + 16; ++q) win[q] = (q < span_w && t0 + q < span) ? stage[t0 + q] : 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int q = 0; q < 17; ++q)
            if (q <= 2 * half) sums[u] += win[u + q];
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u)
          for (int q = 0; q <= 2 * half; ++q)
            if (t0 + u + q < span) sums[u] += stage[t0 + u + q];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = t0 + u;
        const bool in = t < nseg;
        if (in) {
          v[t] = sums[u];
          if (gvals) gvals[s0 + t] = (a.pool == 1) ? sums[u] : sums[u] / pool_div;
        }
        if (need_rank) hist_add(sh.rx.hist[0], order_key(sums[u]) >> 21, in);
      }
    }
  } else {
    // long rows: pooled values go straight to global memory (L2-resident)
    for (int base = 0; base < nseg; base += kThreads) {
      const int t = base + threadIdx.x;
      const bool in = t < nseg;
      float val = 0.f;
      if (in) {
        float sum = 0.f;
        for (int q = -half; q <= half; ++q) {
          const int64_t pos = s0 + t + q;
          if (pos < 0 || pos >= L) continue;
          float rs = 0.f;
          for (int r = 0; r < a.row_group; ++r) rs += rows0[(int64_t)r * a.row_stride + pos];
          sum += rs;
        }
        val = sum;  // ranked as the pooled sum (see the shared-memory path)
        v[t] = val;
      }
      if (need_rank) hist_add(sh.rx.hist[0], order_key(val) >> 21, in);
    }
  }
  // global-memory mode keeps the pooled sums in the caller's buffer while
  // ranking; it holds the averages once this CTA no longer reads them
  auto finish_gvals = [&]() {
    if (!a.smem_vals && gvals && a.pool > 1) {
      __syncthreads();
      for (int t = threadIdx.x; t < nseg; t += kThreads) v[t] = v[t] / pool_div;
    }
  };
  if (!need_rank) {
    finish_gvals();
    return;
  }

  // ---- radix passes ---------------------------------------------------------
  cluster.sync();
  cluster_find_bucket(cluster, sh.rx, 0, kBins, (uint32_t)kk);
  const uint32_t b1 = sh.rx.found_bucket;
  uint32_t want = sh.rx.found_rem;
  // keys of this CTA above bucket b1 are selected whatever the finer bits
  const uint32_t gt1 = local_count_above(sh.rx, 0, kBins, b1);

  for (int i = threadIdx.x; i < kBins; i += kThreads) sh.rx.hist[1][i] = 0;
  __syncthreads();
  for (int base = 0; base < nseg; base += kThreads) {
    const int t = base + threadIdx.x;
    const uint32_t key = t < nseg ? order_key(v[t]) : 0u;
    hist_add(sh.rx.hist[1], (key >> 10) & 2047u, t < nseg && (key >> 21) == b1);
  }
  cluster.sync();
  cluster_find_bucket(cluster, sh.rx, 1, kBins, want);
  const uint32_t b2 = sh.rx.found_bucket;
  want = sh.rx.found_rem;
  const uint32_t pre2 = (b1 << 11) | b2;
  const uint32_t gt2 = local_count_above(sh.rx, 1, kBins, b2);

  for (int i = threadIdx.x; i < kBins; i += kThreads) sh.rx.hist[0][i] = 0;
  __syncthreads();
  for (int base = 0; base < nseg; base += kThreads) {
    const int t = base + threadIdx.x;
    const uint32_t key = t < nseg ? order_key(v[t]) : 0u;
    hist_add(sh.rx.hist[0], key & 1023u, t < nseg && (key >> 10) == pre2);
  }
  cluster.sync();
  cluster_find_bucket(cluster, sh.rx, 0, 1024, want);
  const uint32_t b3 = sh.rx.found_bucket;
  const uint32_t T = (pre2 << 10) | b3;
  const uint32_t need_eq = sh.rx.found_rem;  // how many keys == T are taken (lowest positions)

  // ---- counts per CTA (from the local histograms), then cluster prefix ------
  const uint32_t gt3 = local_count_above(sh.rx, 0, 1024, b3);
  if (threadIdx.x == 0) {
    sh.cnt_gt = gt1 + gt2 + gt3;
    sh.cnt_eq = (uint32_t)sh.rx.hist[0][b3];
  }
  cluster.sync();
  uint32_t out_base = 0, eq_seen = 0;
  if (threadIdx.x < 32) {
    // lanes c < crank hold rank c's counts; a warp scan gives this CTA's offset
    const int lane = threadIdx.x;
    uint32_t cg_ = 0, ce = 0;
    if (lane < crank) {
      const SelShared* r = cluster.map_shared_rank(&sh, lane);
      cg_ = r->cnt_gt;
      ce = r->cnt_eq;
    }
    // equal keys are taken by rank order: rank c takes min(ce, quota left)
    uint32_t ce_before = ce;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, ce_before, o);
      if (lane >= o) ce_before += y;
    }
    ce_before -= ce;  // exclusive
    const uint32_t take = ce_before < need_eq ? min(need_eq - ce_before, ce) : 0u;
    uint32_t sum = cg_ + take;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    uint32_t eqs = ce;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) eqs += __shfl_xor_sync(0xffffffffu, eqs, o);
    if (lane == 0) {
      sh.rx.found_bucket = sum;  // reused as scratch: output offset of this CTA
      sh.rx.found_rem = eqs;     // equal keys in earlier ranks
    }
  }
  __syncthreads();
  out_base = sh.rx.found_bucket;
  eq_seen = sh.rx.found_rem;

  // ---- order-preserving compaction -----------------------------------------
  for (int t0 = 0; t0 < nseg; t0 += kThreads * kPerTile) {
    const int tb = t0 + threadIdx.x * kPerTile;
    uint32_t keys[kPerTile];
    uint32_t my_gt = 0, my_eq = 0;
    if (a.smem_vals && tb + kPerTile <= nseg) {
      const float4 f = *reinterpret_cast<const float4*>(v + tb);  // conflict-free 16-B loads
      keys[0] = order_key(f.x);
      keys[1] = order_key(f.y);
      keys[2] = order_key(f.z);
      keys[3] = order_key(f.w);
    } else {
#pragma unroll
      for (int q = 0; q < kPerTile; ++q) keys[q] = (tb + q < nseg) ? order_key(v[tb + q]) : 0u;
    }
#pragma unroll
    for (int q = 0; q < kPerTile; ++q) {
      if (tb + q < nseg) {
        my_gt += keys[q] > T;
        my_eq += keys[q] == T;
      }
    }
    uint32_t tile_tot;
    const uint32_t pref = block_excl_scan((my_eq << 16) | my_gt, sh.rx.warp_tmp, &tile_tot);
    uint32_t g_before = pref & 0xffffu, e_before = pref >> 16;
    const uint32_t quota = eq_seen < need_eq ? need_eq - eq_seen : 0u;
#pragma unroll
    for (int q = 0; q < kPerTile; ++q) {
      const int t = tb + q;
      if (t >= nseg) break;
      const int32_t j = (int32_t)(s0 + t);
      if (keys[q] > T) {
        out[out_base + g_before + (e_before < quota ? e_before : quota)] = j;
        ++g_before;
      } else if (keys[q] == T) {
        if (e_before < quota) out[out_base + g_before + e_before] = j;
        ++e_before;
      }
    }
    const uint32_t tg = tile_tot & 0xffffu, te = tile_tot >> 16;
    out_base += tg + (te < quota ? te : quota);
    eq_seen += te;
  }
  finish_gvals();
  cluster.sync();  // remote reads of sh are over before any CTA exits
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

  cluster_find_bucket(cluster, sh.rx, 0, kBins, (uint32_t)m);
  const uint32_t b1 = sh.rx.found_bucket;
  uint32_t want = sh.rx.found_rem;
  for (int i = threadIdx.x; i < kBins; i += kThreads) sh.rx.hist[1][i] = 0;
  __syncthreads();
  for (int64_t j = s0 + threadIdx.x; j < s1; j += kThreads) {
    const uint32_t key = order_key(row[j] * a.inv_mass);
    if ((key >> 21) == b1) atomicAdd(&sh.rx.hist[1][(key >> 10) & 2047u], 1);
  }
  cluster.sync();
  cluster_find_bucket(cluster, sh.rx, 1, kBins, want);
  const uint32_t pre2 = (b1 << 11) | sh.rx.found_bucket;
  want = sh.rx.found_rem;
  for (int i = threadIdx.x; i < kBins; i += kThreads) sh.rx.hist[0][i] = 0;
  __syncthreads();
  for (int64_t j = s0 + threadIdx.x; j < s1; j += kThreads) {
    const uint32_t key = order_key(row[j] * a.inv_mass);
    if ((key >> 10) == pre2) atomicAdd(&sh.rx.hist[0][key & 1023u], 1);
  }
  cluster.sync();
  cluster_find_bucket(cluster, sh.rx, 0, 1024, want);
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

constexpr size_t kSelDynMax = 180 * 1024;  // dynamic smem budget for pooled segments

kvc_status launch_select(const SelArgs& a, int out_rows, int batch, int64_t seg, cudaStream_t st) {
  const size_t dyn = sel_dyn_smem(seg, a.pool / 2, a.smem_vals);
  static std::mutex mu;
  static uint64_t done = 0;
  int dev = 0;
  KVC_CUDA_TRY(cudaGetDevice(&dev));
  {
    std::lock_guard<std::mutex> lk(mu);
    if (dev >= 64 || !((done >> dev) & 1)) {
      KVC_CUDA_TRY(cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)kSelDynMax));
      if (dev < 64) done |= (uint64_t)1 << dev;
    }
  }
  dim3 grid(kCS, out_rows, batch);
  select_kernel<<<grid, kThreads, dyn, st>>>(a);
  count_launch();
  KVC_CUDA_TRY(cudaGetLastError());
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
  const int64_t seg = (n - window + kCS - 1) / kCS;
  a.smem_vals = sel_dyn_smem(seg, pool_kernel / 2, true) <= kSelDynMax;
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
  return launch_select(a, out_rows, 1, seg, (cudaStream_t)stream);
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
  const int64_t seg_max = (std::max<int64_t>(max_seqlen, window) - window + kCS - 1) / kCS;
  if (sel_dyn_smem(seg_max, pool_kernel / 2, true) > kSelDynMax &&
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
  const int64_t seg = (std::max<int64_t>(max_seqlen, window) - window + kCS - 1) / kCS;
  a.smem_vals = sel_dyn_smem(seg, pool_kernel / 2, true) <= kSelDynMax;
  a.seg_cap = seg;
  if (!a.smem_vals) a.vals_g = static_cast<float*>(ws);
  return launch_select(a, out_rows, batch, seg, (cudaStream_t)stream);
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
  stats_kernel<<<grid, kThreads, 0, (cudaStream_t)stream>>>(a);
  count_launch();
  KVC_CUDA_TRY(cudaGetLastError());
  return KVC_OK;
}
