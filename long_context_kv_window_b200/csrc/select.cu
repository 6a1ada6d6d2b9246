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

#include "common.cuh"

namespace cg = cooperative_groups;

namespace kvc {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kCS = 8;          // CTAs per ranking row (portable cluster size)
constexpr int kStage = 4096;    // pooled outputs per staging round
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

struct RadixShared {
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

// After every CTA of the cluster filled hist[buf] (and a cluster barrier),
// sum the kCS histograms and find the bin that holds the want-th largest
// candidate: count(bins above) < want <= count(bins above) + tot[bin].
// Bins are visited from the top.  Returns through sh.found_*.
__device__ void cluster_find_bucket(cg::cluster_group& cluster, RadixShared& sh, int buf, int nbins,
                                    uint32_t want) {
  for (int b = threadIdx.x; b < nbins; b += kThreads) {
    int s = 0;
#pragma unroll
    for (int c = 0; c < kCS; ++c) s += cluster.map_shared_rank(&sh.hist[buf][0], c)[b];
    sh.tot[b] = s;
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
  float* vals;             // pooled prefix scores
  int64_t vals_stride;     // per output row
  bool vals_packed;        // vals indexed by packed token offset (varlen / workspace)
  int out_rows;
  int32_t* err;
};

struct SelShared {
  RadixShared rx;
  float stage[kStage + 2 * kMaxHalf];
  uint32_t cnt_gt, cnt_eq;  // this CTA's counts for the output phase
};

__global__ void __cluster_dims__(kCS, 1, 1) __launch_bounds__(kThreads, 1)
select_kernel(const SelArgs a) {
  __shared__ SelShared sh;
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

  // ---- segment of this CTA and the pooled scores --------------------------
  const int64_t seg = (L + kCS - 1) / kCS;
  const int64_t s0 = (int64_t)crank * seg < L ? (int64_t)crank * seg : L;
  const int64_t s1 = s0 + seg < L ? s0 + seg : L;
  const int half = a.pool / 2;
  const float pool_div = (float)a.pool;
  const float* rows0 = a.scores + (int64_t)o * a.row_group * a.row_stride + start;
  float* vals = a.vals + (int64_t)o * a.vals_stride + (a.vals_packed ? start : 0);
  const bool need_rank = (a.k < len) && kk > 0;

  for (int i = threadIdx.x; i < kBins; i += kThreads) sh.rx.hist[0][i] = 0;
  __syncthreads();

  for (int64_t c0 = s0; c0 < s1; c0 += kStage) {
    const int64_t c1 = c0 + kStage < s1 ? c0 + kStage : s1;
    const int64_t lo = c0 - half;
    const int span = (int)(c1 - c0) + 2 * half;
    for (int t = threadIdx.x; t < span; t += kThreads) {
      const int64_t u = lo + t;
      float s = 0.f;
      if (u >= 0 && u < L) {
        for (int r = 0; r < a.row_group; ++r) s += rows0[(int64_t)r * a.row_stride + u];
      }
      sh.stage[t] = s;
    }
    __syncthreads();
    for (int t = threadIdx.x; t < (int)(c1 - c0); t += kThreads) {
      float v;
      if (a.pool == 1) {
        v = sh.stage[t];
      } else {
        float s = 0.f;
        for (int q = 0; q <= 2 * half; ++q) s += sh.stage[t + q];
        v = s / pool_div;
      }
      vals[c0 + t] = v;  // pooled scores are always materialised
      if (need_rank) atomicAdd(&sh.rx.hist[0][order_key(v) >> 21], 1);
    }
    __syncthreads();
  }
  if (!need_rank) {
    cluster.sync();  // keep every CTA resident until the cluster is done
    return;
  }

  // ---- radix passes ---------------------------------------------------------
  cluster.sync();
  cluster_find_bucket(cluster, sh.rx, 0, kBins, (uint32_t)kk);
  const uint32_t b1 = sh.rx.found_bucket;
  uint32_t want = sh.rx.found_rem;

  for (int i = threadIdx.x; i < kBins; i += kThreads) sh.rx.hist[1][i] = 0;
  __syncthreads();
  for (int64_t j = s0 + threadIdx.x; j < s1; j += kThreads) {
    const uint32_t key = order_key(vals[j]);
    if ((key >> 21) == b1) atomicAdd(&sh.rx.hist[1][(key >> 10) & 2047u], 1);
  }
  cluster.sync();
  cluster_find_bucket(cluster, sh.rx, 1, kBins, want);
  const uint32_t b2 = sh.rx.found_bucket;
  want = sh.rx.found_rem;
  const uint32_t pre2 = (b1 << 11) | b2;

  for (int i = threadIdx.x; i < kBins; i += kThreads) sh.rx.hist[0][i] = 0;
  __syncthreads();
  for (int64_t j = s0 + threadIdx.x; j < s1; j += kThreads) {
    const uint32_t key = order_key(vals[j]);
    if ((key >> 10) == pre2) atomicAdd(&sh.rx.hist[0][key & 1023u], 1);
  }
  cluster.sync();
  cluster_find_bucket(cluster, sh.rx, 0, 1024, want);
  const uint32_t T = (pre2 << 10) | sh.rx.found_bucket;
  const uint32_t need_eq = sh.rx.found_rem;  // how many keys == T are taken (lowest positions)

  // ---- counts per CTA, then cluster prefix ---------------------------------
  uint32_t gt = 0, eq = 0;
  for (int64_t j = s0 + threadIdx.x; j < s1; j += kThreads) {
    const uint32_t key = order_key(vals[j]);
    gt += key > T;
    eq += key == T;
  }
  uint32_t tot;
  block_excl_scan(gt, sh.rx.warp_tmp, &tot);
  if (threadIdx.x == 0) sh.cnt_gt = tot;
  block_excl_scan(eq, sh.rx.warp_tmp, &tot);
  if (threadIdx.x == 0) sh.cnt_eq = tot;
  cluster.sync();
  uint32_t out_base = 0, eq_seen = 0;
  for (int c = 0; c < crank; ++c) {
    SelShared* r = cluster.map_shared_rank(&sh, c);
    const uint32_t e = r->cnt_eq;
    const uint32_t take = eq_seen < need_eq ? (need_eq - eq_seen < e ? need_eq - eq_seen : e) : 0u;
    out_base += r->cnt_gt + take;
    eq_seen += e;
  }

  // ---- order-preserving compaction -----------------------------------------
  for (int64_t t0 = s0; t0 < s1; t0 += (int64_t)kThreads * kPerTile) {
    const int64_t j0 = t0 + (int64_t)threadIdx.x * kPerTile;
    uint32_t keys[kPerTile];
    uint32_t my_gt = 0, my_eq = 0;
#pragma unroll
    for (int q = 0; q < kPerTile; ++q) {
      const int64_t j = j0 + q;
      keys[q] = (j < s1) ? order_key(vals[j]) : 0u;
      if (j < s1) {
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
      const int64_t j = j0 + q;
      if (j >= s1) break;
      if (keys[q] > T) {
        out[out_base + g_before + (e_before < quota ? e_before : quota)] = (int32_t)j;
        ++g_before;
      } else if (keys[q] == T) {
        if (e_before < quota) out[out_base + g_before + e_before] = (int32_t)j;
        ++e_before;
      }
    }
    const uint32_t tg = tile_tot & 0xffffu, te = tile_tot >> 16;
    out_base += tg + (te < quota ? te : quota);
    eq_seen += te;
  }
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
  if (pooled) {
    a.vals = pooled;
    a.vals_stride = n - window;
    a.vals_packed = false;
  } else {
    size_t need = 0;
    kvc_select_workspace_size(out_rows, 1, n, &need);
    if (!ws || ws_bytes < need || !aligned(ws, kWsAlign))
      return fail(KVC_ERR_WORKSPACE, "select workspace missing, too small or not 256-B aligned");
    a.vals = static_cast<float*>(ws);
    a.vals_stride = n;
    a.vals_packed = true;
  }
  dim3 grid(kCS, out_rows, 1);
  select_kernel<<<grid, kThreads, 0, (cudaStream_t)stream>>>(a);
  count_launch();
  KVC_CUDA_TRY(cudaGetLastError());
  return KVC_OK;
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
  if (!ws || ws_bytes < need || !aligned(ws, kWsAlign))
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
  a.vals = static_cast<float*>(ws);
  a.vals_stride = total;
  a.vals_packed = true;
  a.out_rows = out_rows;
  a.err = dev_err;
  dim3 grid(kCS, out_rows, batch);
  select_kernel<<<grid, kThreads, 0, (cudaStream_t)stream>>>(a);
  count_launch();
  KVC_CUDA_TRY(cudaGetLastError());
  return KVC_OK;
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
