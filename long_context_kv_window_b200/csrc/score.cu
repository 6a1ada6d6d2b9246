// score.cu -- observation-window attention aggregate on tcgen05 tensor cores.
//
// FastKV (gist.science 2502.01068) section 2.A: token importance at the TSP
// layer is the attention paid to each context token by a window of recent
// queries.  FastKV abstract: GQA-aware, i.e. one aggregate per KV head over
// the query heads of its group.  StructKV (gist.science 2604.06746) section
// 2.A: C_global accumulates the per-layer contributions (`accum`).
//
// For KV head g the G*w window rows (query head of the group x window query)
// form a dense R x d operand, so Q_win * K^T is a real contraction and runs
// on tcgen05 (bf16 in, fp32 accumulation in TMEM).  The softmax normaliser
// of a row needs all N keys before any probability is known, so the
// aggregate takes two passes over K:
//   pass 1 (rows on the MMA M axis, keys on N): each epilogue thread owns one
//          row and keeps an online max / sum of 2^(s*log2e - max) over its
//          chunk of keys and writes that chunk partial to the workspace;
//   pass 2 (keys on M, rows on N): the epilogue first combines the chunk
//          partials of its (sequence, head) into one bias
//          b_r = max_r + log2(sum_r) per row, while TMA and MMA already run;
//          then each epilogue thread owns one key and sums 2^(s*log2e - b_r)
//          over the rows -- a thread-local reduction.
// Both passes stream the same K tiles (TMA, 128-byte swizzle) into a
// multi-stage shared-memory ring; heads are processed in groups whose K fits
// in L2, so pass 2 re-reads K from L2 rather than HBM.
//
// Warp roles per CTA: warp 0 issues TMA, warp 1 allocates TMEM and issues
// MMAs, warps 2..5 drain TMEM (epilogue).  Every wait is bounded; on a
// timeout the CTA records KVC_DEV_ERR_TIMEOUT, lets in-flight copies and MMAs
// land, frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "tc.cuh"

namespace kvc {
namespace {

constexpr int kTile = 128;  // keys per tile
constexpr int kStages = 4;
constexpr int kEpiWarps = 4;
constexpr int kThreadsScore = 64 + 32 * kEpiWarps;
constexpr int kMinChunkTiles = 4;
constexpr double kLog2e = 1.4426950408889634;

struct ScoreArgs {
  const uint16_t* q;
  int64_t q_sb, q_sw, q_sh;  // Q_win strides (elements): sequence, window row, head
  const int32_t* cu;         // nullptr: one sequence of n tokens
  int64_t n;                 // single-sequence length (ignored with cu)
  int B;
  int Hkv, G, w, R, Rq, Rn;  // rows per KV head, rows in smem, MMA N (pass 2)
  int nb1;                   // 128-row blocks in pass 1
  int acc_stride1;           // pass 1: TMEM columns between the two accumulator buffers
  int acc_stride;            // pass 2: TMEM columns between the two accumulator buffers
  uint32_t tmem_cols;        // TMEM columns allocated
  int g0;                    // first KV head of this launch
  int chunk_keys;
  int max_chunks;            // partial slots per KV head
  float c;                   // scale * log2(e)
  float* part_m;             // [Hkv][max_chunks][Rq]
  double* part_l;            // [Hkv][max_chunks][Rq]
  float* scores;             // [Hkv][total]
  float* accum;              // [Hkv][total] or nullptr
  int64_t total;
  int32_t* err;
};

struct Work {
  int b;
  int chunk;       // chunk index inside the sequence
  int gid;         // global chunk index (partial slot)
  int nchunks;     // chunks of this sequence
  int64_t start;   // first packed token of the sequence
  int64_t len;
  bool valid;
  bool bad;
};

// Map a linear chunk index onto (sequence, chunk).  Malformed sequences
// (non-monotone cu_seqlens or shorter than the window) own one chunk each.
__device__ __forceinline__ Work map_work(const ScoreArgs& a, int linear) {
  int base = 0;
  for (int b = 0; b < a.B; ++b) {
    const SeqSpan s = seq_span(a.cu, b, a.n);
    const bool bad = s.start < 0 || s.len < a.w || s.start + s.len > a.total;
    const int nch = bad ? 1 : (int)((s.len + a.chunk_keys - 1) / a.chunk_keys);
    if (linear < base + nch) return Work{b, linear - base, linear, nch, s.start, s.len, true, bad};
    base += nch;
  }
  return Work{0, 0, 0, 0, 0, 0, false, false};
}

template <int D>
struct Smem {
  static constexpr int kChunks = D / 64;            // 64-element (128 B) swizzle columns
  static constexpr int kStageBytes = kChunks * kTile * 128;
  __host__ __device__ static size_t q_bytes(int Rq) { return (size_t)kChunks * Rq * 128; }
  __host__ __device__ static size_t total(int Rq) {
    return 1024 /*alignment slack*/ + q_bytes(Rq) + (size_t)kStages * kStageBytes + 256 /*barriers*/ +
           (size_t)Rq * sizeof(float) /*bias*/ + 64;
  }
};

struct Barriers {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint32_t tmem_base;
  int abort;
};

// Q rows of KV head g into the K-major 128-byte swizzled layout; rows past R
// are zero.  Row r = i*G + h_local (window row i, query head g*G + h_local).
template <int D>
__device__ __forceinline__ void load_q_swizzled(const ScoreArgs& a, int b, int g, uint8_t* qs) {
  constexpr int kChunks = D / 64;
  const int nvec = a.Rq * kChunks * 8;
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    const int j = v & 7;
    const int r = (v >> 3) % a.Rq;
    const int c = (v >> 3) / a.Rq;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (r < a.R) {
      const int i = r / a.G, hl = r % a.G;
      const uint16_t* src =
          a.q + (int64_t)b * a.q_sb + (int64_t)i * a.q_sw + (int64_t)(g * a.G + hl) * a.q_sh + c * 64 + j * 8;
      val = *reinterpret_cast<const uint4*>(src);
    }
    *reinterpret_cast<uint4*>(qs + (size_t)c * a.Rq * 128 + (size_t)r * 128 + ((j ^ (r & 7)) << 4)) = val;
  }
  tc::fence_proxy_async_smem();
}

// Producer: stream the chunk's K tiles of head g into the stage ring.
template <int D>
__device__ __forceinline__ void produce(const void* kmap, Barriers* bars, uint8_t* kst, int g, int64_t row0,
                                        int ntiles) {
  constexpr int kChunks = D / 64;
  constexpr uint32_t kBytes = (uint32_t)Smem<D>::kStageBytes;
  int issued = 0;
  for (int t = 0; t < ntiles; ++t) {
    const int s = t % kStages;
    const int u = t / kStages;
    if (u > 0 && !tc::mbar_wait(&bars->empty[s], (u - 1) & 1, &bars->abort)) break;
    tc::mbar_arrive_expect_tx(&bars->full[s], kBytes);
    uint8_t* dst = kst + (size_t)s * Smem<D>::kStageBytes;
#pragma unroll
    for (int c = 0; c < kChunks; ++c)
      tc::tma_load_3d(dst + c * kTile * 128, kmap, &bars->full[s], c * 64, g, (int)(row0 + (int64_t)t * kTile));
    issued = t + 1;
  }
  if (bars->abort) {
    // let every copy already issued land before the CTA can exit
    for (int t = std::max(0, issued - kStages); t < issued; ++t)
      tc::mbar_drain(&bars->full[t % kStages], (t / kStages) & 1);
  }
}

__device__ __forceinline__ void record_timeout(int32_t* err) { set_dev_err(err, KVC_DEV_ERR_TIMEOUT); }

// --------------------------------------------------------------------------
// pass 1: per-row max / sum over a chunk of keys
// --------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kThreadsScore, 1)
score_pass1_kernel(const __grid_constant__ CUtensorMap kmap, const ScoreArgs a) {
  constexpr int kChunks = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qs = smem;
  uint8_t* kst = qs + Smem<D>::q_bytes(a.Rq);
  Barriers* bars = reinterpret_cast<Barriers*>(kst + (size_t)kStages * Smem<D>::kStageBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = a.g0 + blockIdx.y;
  const Work wk = map_work(a, blockIdx.x);
  if (!wk.valid) return;
  if (wk.bad) {
    if (threadIdx.x == 0 && blockIdx.y == 0) set_dev_err(a.err, KVC_DEV_ERR_SEQLENS);
    return;
  }
  const int64_t k0 = (int64_t)wk.chunk * a.chunk_keys;
  const int64_t k1 = std::min<int64_t>(wk.len, k0 + a.chunk_keys);
  const int ntiles = (int)((k1 - k0 + kTile - 1) / kTile);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&bars->full[s], 1);
      tc::mbar_init(&bars->empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->tfull[s], 1);
      tc::mbar_init(&bars->tempty[s], kEpiWarps);
    }
    bars->abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) tc::prefetch_tmap(&kmap);
  if (warp == 1) {
    tc::tmem_alloc(&bars->tmem_base, a.tmem_cols);
    tc::tmem_relinquish();
  }
  load_q_swizzled<D>(a, wk.b, g, qs);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0) produce<D>(&kmap, bars, kst, g, wk.start + k0, ntiles);
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(128, kTile);
      const uint32_t qbase = tc::smem_u32(qs), kbase = tc::smem_u32(kst);
      int t = 0;
      for (; t < ntiles; ++t) {
        const int s = t % kStages, acc = t & 1;
        if (!tc::mbar_wait(&bars->full[s], (t / kStages) & 1, &bars->abort)) break;
        if (t >= 2 && !tc::mbar_wait(&bars->tempty[acc], ((t >> 1) - 1) & 1, &bars->abort)) break;
        tc::tc_fence_after();
        for (int mb = 0; mb < a.nb1; ++mb) {
          const uint32_t d = tmem + (uint32_t)(acc * a.acc_stride1 + mb * kTile);
#pragma unroll
          for (int c = 0; c < kChunks; ++c)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              const uint64_t ad = tc::desc_k_sw128(qbase + (uint32_t)(c * a.Rq * 128 + mb * kTile * 128 + ks * 32));
              const uint64_t bd = tc::desc_k_sw128(kbase + (uint32_t)(s * Smem<D>::kStageBytes + c * kTile * 128 + ks * 32));
              tc::mma_bf16(d, ad, bd, idesc, (c | ks) != 0);
            }
        }
        tc::mma_commit(&bars->empty[s]);
        tc::mma_commit(&bars->tfull[acc]);
      }
      if (t > 0) tc::mbar_drain(&bars->tfull[(t - 1) & 1], ((t - 1) >> 1) & 1);  // last MMAs landed
    }
  } else {
    // ---- epilogue: one row per thread and row block --------------------------
    const int q = warp & 3;
    const int rl = 32 * q + lane;  // lane within a 128-row block
    float m_run[2] = {-INFINITY, -INFINITY};
    double l_run[2] = {0.0, 0.0};
    const int64_t first_window_key = wk.len - a.w;  // earliest window row sees keys <= this
    for (int t = 0; t < ntiles; ++t) {
      const int acc = t & 1;
      if (!tc::mbar_wait(&bars->tfull[acc], (t >> 1) & 1, &bars->abort)) break;
      tc::tc_fence_after();
      const int64_t j0 = k0 + (int64_t)t * kTile;  // first key of the tile (sequence-local)
#pragma unroll
      for (int mb = 0; mb < 2; ++mb) {
        if (mb >= a.nb1) break;
        uint32_t x[4][32];
        const uint32_t base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * a.acc_stride1 + mb * kTile);
        KVC_TMEM_LD32(base + 0, x[0]);
        KVC_TMEM_LD32(base + 32, x[1]);
        KVC_TMEM_LD32(base + 64, x[2]);
        KVC_TMEM_LD32(base + 96, x[3]);
        KVC_TMEM_WAIT_LD32(x[0]);
        KVC_TMEM_TIE32(x[1]);
        KVC_TMEM_TIE32(x[2]);
        KVC_TMEM_TIE32(x[3]);
        if (mb == a.nb1 - 1) {
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&bars->tempty[acc]);
        }
        const int r = mb * kTile + rl;
        if (r >= a.R) continue;
        const bool full_tile = (j0 + kTile - 1 <= first_window_key);
        if (!full_tile) {
          // keys past this row's own position (or past the sequence) are masked to -inf
          const int64_t last_key = first_window_key + r / a.G;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (j0 + cc * 32 + e > last_key) x[cc][e] = __float_as_uint(-INFINITY);
        }
        float t4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
          for (int e = 0; e < 32; ++e) t4[e & 3] = fmaxf(t4[e & 3], __uint_as_float(x[cc][e]));
        const float tmax = fmaxf(fmaxf(t4[0], t4[1]), fmaxf(t4[2], t4[3]));
        if (tmax == -INFINITY) continue;
        const float ynew = tmax * a.c;
        if (ynew > m_run[mb]) {
          l_run[mb] *= (double)exp2f(m_run[mb] - ynew);
          m_run[mb] = ynew;
        }
        const float mneg = -m_run[mb];
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
          for (int e = 0; e < 32; ++e) s4[e & 3] += tc::ex2_approx(fmaf(__uint_as_float(x[cc][e]), a.c, mneg));
        l_run[mb] += (double)((s4[0] + s4[1]) + (s4[2] + s4[3]));
      }
    }
    // ---- chunk partials (combined by pass 2) ----------------------------------
    if (!bars->abort) {
#pragma unroll
      for (int mb = 0; mb < 2; ++mb) {
        if (mb >= a.nb1) break;
        const int r = mb * kTile + rl;
        if (r >= a.R) continue;
        const size_t slot = ((size_t)g * a.max_chunks + wk.gid) * a.Rq + r;
        a.part_m[slot] = m_run[mb];
        a.part_l[slot] = l_run[mb];
      }
    }
  }
  __syncthreads();
  if (bars->abort && threadIdx.x == 0) record_timeout(a.err);
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, a.tmem_cols);
  }
}

// --------------------------------------------------------------------------
// pass 2: per-key sum of normalised probabilities over the window rows
// --------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kThreadsScore, 1)
score_pass2_kernel(const __grid_constant__ CUtensorMap kmap, const ScoreArgs a) {
  constexpr int kChunks = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qs = smem;
  uint8_t* kst = qs + Smem<D>::q_bytes(a.Rq);
  Barriers* bars = reinterpret_cast<Barriers*>(kst + (size_t)kStages * Smem<D>::kStageBytes);
  float* bias_s = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = a.g0 + blockIdx.y;
  const Work wk = map_work(a, blockIdx.x);
  if (!wk.valid) return;
  if (wk.bad) {
    // leave nothing stale behind: zero whatever part of the row is addressable
    if (wk.start >= 0 && wk.len > 0 && wk.start + wk.len <= a.total)
      for (int64_t j = threadIdx.x; j < wk.len; j += blockDim.x) a.scores[(int64_t)g * a.total + wk.start + j] = 0.f;
    return;
  }
  const int64_t k0 = (int64_t)wk.chunk * a.chunk_keys;
  const int64_t k1 = std::min<int64_t>(wk.len, k0 + a.chunk_keys);
  const int ntiles = (int)((k1 - k0 + kTile - 1) / kTile);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&bars->full[s], 1);
      tc::mbar_init(&bars->empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->tfull[s], 1);
      tc::mbar_init(&bars->tempty[s], kEpiWarps);
    }
    bars->abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) tc::prefetch_tmap(&kmap);
  if (warp == 1) {
    tc::tmem_alloc(&bars->tmem_base, a.tmem_cols);
    tc::tmem_relinquish();
  }
  load_q_swizzled<D>(a, wk.b, g, qs);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0) produce<D>(&kmap, bars, kst, g, wk.start + k0, ntiles);
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(128, a.Rn);
      const uint32_t qbase = tc::smem_u32(qs), kbase = tc::smem_u32(kst);
      int t = 0;
      for (; t < ntiles; ++t) {
        const int s = t % kStages, acc = t & 1;
        if (!tc::mbar_wait(&bars->full[s], (t / kStages) & 1, &bars->abort)) break;
        if (t >= 2 && !tc::mbar_wait(&bars->tempty[acc], ((t >> 1) - 1) & 1, &bars->abort)) break;
        tc::tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * a.acc_stride);
#pragma unroll
        for (int c = 0; c < kChunks; ++c)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t ad = tc::desc_k_sw128(kbase + (uint32_t)(s * Smem<D>::kStageBytes + c * kTile * 128 + ks * 32));
            const uint64_t bd = tc::desc_k_sw128(qbase + (uint32_t)(c * a.Rq * 128 + ks * 32));
            tc::mma_bf16(d, ad, bd, idesc, (c | ks) != 0);
          }
        tc::mma_commit(&bars->empty[s]);
        tc::mma_commit(&bars->tfull[acc]);
      }
      if (t > 0) tc::mbar_drain(&bars->tfull[(t - 1) & 1], ((t - 1) >> 1) & 1);
    }
  } else {
    // ---- epilogue prologue: per-row bias from the pass-1 chunk partials --------
    // b_r = M + log2(sum_c l_c 2^(m_c - M)), M = max_c m_c.  Padded columns get
    // b = +inf, so 2^(x*c - inf) = 0 needs no mask.  The producer and MMA warps
    // are already filling the pipeline meanwhile.
    {
      const int et = threadIdx.x - 64;  // 0..127
      const size_t base_slot = ((size_t)g * a.max_chunks + (wk.gid - wk.chunk)) * a.Rq;
      for (int r = et; r < a.Rn; r += 32 * kEpiWarps) {
        if (r >= a.R) {
          bias_s[r] = INFINITY;
          continue;
        }
        constexpr int kB = 8;
        float mx = -INFINITY;
        for (int c0 = 0; c0 < wk.nchunks; c0 += kB) {
          float mv[kB];
#pragma unroll
          for (int u = 0; u < kB; ++u)
            mv[u] = (c0 + u < wk.nchunks) ? __ldcg(&a.part_m[base_slot + (size_t)(c0 + u) * a.Rq + r]) : -INFINITY;
#pragma unroll
          for (int u = 0; u < kB; ++u) mx = fmaxf(mx, mv[u]);
        }
        double l = 0.0;
        for (int c0 = 0; c0 < wk.nchunks; c0 += kB) {
          float mv[kB];
          double lv[kB];
#pragma unroll
          for (int u = 0; u < kB; ++u) {
            const bool in = c0 + u < wk.nchunks;
            mv[u] = in ? __ldcg(&a.part_m[base_slot + (size_t)(c0 + u) * a.Rq + r]) : -INFINITY;
            lv[u] = in ? __ldcg(&a.part_l[base_slot + (size_t)(c0 + u) * a.Rq + r]) : 0.0;
          }
#pragma unroll
          for (int u = 0; u < kB; ++u)
            if (mv[u] != -INFINITY) l += lv[u] * (double)exp2f(mv[u] - mx);
        }
        bias_s[r] = (float)((double)mx + log2(l));
      }
      tc::named_bar_sync(1, 32 * kEpiWarps);
    }
    // ---- epilogue: one key per thread ------------------------------------------
    const int q = warp & 3;
    const int kl = 32 * q + lane;              // key within the tile
    const int64_t first_window_key = wk.len - a.w;
    const int ngroups = (a.Rn + 127) / 128;    // groups of up to 4 x 32 columns
    for (int t = 0; t < ntiles; ++t) {
      const int acc = t & 1;
      if (!tc::mbar_wait(&bars->tfull[acc], (t >> 1) & 1, &bars->abort)) break;
      tc::tc_fence_after();
      const int64_t j = k0 + (int64_t)t * kTile + kl;  // this thread's key (sequence-local)
      const bool masked_tile = (k0 + (int64_t)t * kTile + kTile - 1 > first_window_key);
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
      for (int grp = 0; grp < ngroups; ++grp) {
        const int col0 = grp * 128;
        const int ncol = min(128, a.Rn - col0);  // multiple of 16
        const int nfull = ncol >> 5;             // whole 32-column chunks (0..4)
        const bool tail16 = (ncol & 31) != 0;    // one trailing 16-column chunk
        uint32_t x[4][32];
        uint32_t xt[32];
        const uint32_t base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * a.acc_stride + col0);
        if (nfull > 0) KVC_TMEM_LD32(base + 0, x[0]);
        if (nfull > 1) KVC_TMEM_LD32(base + 32, x[1]);
        if (nfull > 2) KVC_TMEM_LD32(base + 64, x[2]);
        if (nfull > 3) KVC_TMEM_LD32(base + 96, x[3]);
        if (tail16) KVC_TMEM_LD16(base + 32 * nfull, xt);
        KVC_TMEM_WAIT_LD32(x[0]);
        KVC_TMEM_TIE32(x[1]);
        KVC_TMEM_TIE32(x[2]);
        KVC_TMEM_TIE32(x[3]);
        KVC_TMEM_TIE32(xt);
        if (grp == ngroups - 1) {
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&bars->tempty[acc]);
        }
        if (masked_tile) {
          // window rows see only keys up to their own position; later keys (and
          // keys past the sequence) get logit -inf, i.e. probability 0
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            if (cc >= nfull) break;
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (j > first_window_key + (col0 + cc * 32 + e) / a.G) x[cc][e] = __float_as_uint(-INFINITY);
          }
          if (tail16) {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              if (j > first_window_key + (col0 + nfull * 32 + e) / a.G) xt[e] = __float_as_uint(-INFINITY);
          }
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          if (cc >= nfull) break;
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 bb = *reinterpret_cast<const float4*>(&bias_s[col0 + cc * 32 + e]);
            s4[0] += tc::ex2_approx(fmaf(__uint_as_float(x[cc][e + 0]), a.c, -bb.x));
            s4[1] += tc::ex2_approx(fmaf(__uint_as_float(x[cc][e + 1]), a.c, -bb.y));
            s4[2] += tc::ex2_approx(fmaf(__uint_as_float(x[cc][e + 2]), a.c, -bb.z));
            s4[3] += tc::ex2_approx(fmaf(__uint_as_float(x[cc][e + 3]), a.c, -bb.w));
          }
        }
        if (tail16) {
#pragma unroll
          for (int e = 0; e < 16; e += 4) {
            const float4 bb = *reinterpret_cast<const float4*>(&bias_s[col0 + nfull * 32 + e]);
            s4[0] += tc::ex2_approx(fmaf(__uint_as_float(xt[e + 0]), a.c, -bb.x));
            s4[1] += tc::ex2_approx(fmaf(__uint_as_float(xt[e + 1]), a.c, -bb.y));
            s4[2] += tc::ex2_approx(fmaf(__uint_as_float(xt[e + 2]), a.c, -bb.z));
            s4[3] += tc::ex2_approx(fmaf(__uint_as_float(xt[e + 3]), a.c, -bb.w));
          }
        }
      }
      if (j < k1) {
        const float v = (s4[0] + s4[1]) + (s4[2] + s4[3]);
        const int64_t o = (int64_t)g * a.total + wk.start + j;
        a.scores[o] = v;
        if (a.accum) a.accum[o] += v;
      }
    }
  }
  __syncthreads();
  if (bars->abort && threadIdx.x == 0) record_timeout(a.err);
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, a.tmem_cols);
  }
}

// TSP aggregate: tsp[j] = sum_g scores[g][j] (all heads, one row).
__global__ void tsp_sum_kernel(const float* __restrict__ scores, int Hkv, int64_t total, float* __restrict__ tsp) {
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < total; j += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int g = 0; g < Hkv; ++g) s += scores[(int64_t)g * total + j];
    tsp[j] = s;
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

struct Geometry {
  int G, R, Rq, Rn, nb1, acc_stride1, acc_stride;
  uint32_t cols1, cols2;  // TMEM columns for pass 1 / pass 2
};

uint32_t pow2_cols(int c) {
  uint32_t p = 32;
  while ((int)p < c) p <<= 1;
  return p;
}

Geometry geometry(const kvc_score_params* p) {
  Geometry g{};
  g.G = p->num_heads / p->num_kv_heads;
  g.R = g.G * p->window;
  g.Rn = (g.R + 15) / 16 * 16;
  g.nb1 = (g.R + kTile - 1) / kTile;
  g.Rq = std::max(g.nb1 * kTile, g.Rn);
  g.acc_stride1 = g.nb1 * kTile;
  g.acc_stride = (g.Rn + 31) / 32 * 32;
  g.cols1 = pow2_cols(2 * g.nb1 * kTile);
  g.cols2 = pow2_cols(2 * g.acc_stride);
  return g;
}

int max_chunks_bound(int64_t total, int B) { return (int)(total / (kMinChunkTiles * kTile)) + B + 1; }

kvc_status check_params(const kvc_score_params* p) {
  KVC_CHECK_ARG(p != nullptr, "params must be non-NULL");
  KVC_CHECK_ARG(p->num_heads >= 1 && p->num_kv_heads >= 1 && p->num_heads % p->num_kv_heads == 0,
                "num_heads must be a positive multiple of num_kv_heads");
  if (p->head_dim != 64 && p->head_dim != 128) return fail(KVC_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  KVC_CHECK_ARG(p->window >= 1, "window must be >= 1");
  KVC_CHECK_ARG(p->scale > 0.f && p->scale < 1e30f, "scale must be positive and finite");
  const int G = p->num_heads / p->num_kv_heads;
  if ((int64_t)G * p->window > 256) return fail(KVC_ERR_UNSUPPORTED, "G * window must be <= 256");
  return KVC_OK;
}

size_t score_ws_bytes(const kvc_score_params* p, int B, int64_t total) {
  const Geometry gm = geometry(p);
  const int mc = max_chunks_bound(total, B);
  size_t s = kWsAlign;                                                              // reserved
  s += round_up((size_t)p->num_kv_heads * mc * gm.Rq * sizeof(float), kWsAlign);    // part_m
  s += round_up((size_t)p->num_kv_heads * mc * gm.Rq * sizeof(double), kWsAlign);   // part_l
  return s;
}

// The dynamic shared-memory limit is a per-device function attribute.
template <int D>
kvc_status set_smem_attrs(size_t bytes) {
  if (bytes > 227 * 1024) return fail(KVC_ERR_UNSUPPORTED, "score kernel shared memory above 227 KB");
  static std::mutex mu;
  static uint64_t done = 0;  // bit per device ordinal (< 64)
  int dev = 0;
  KVC_CUDA_TRY(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(mu);
  if (dev < 64 && (done >> dev) & 1) return KVC_OK;
  KVC_CUDA_TRY(cudaFuncSetAttribute(score_pass1_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024));
  KVC_CUDA_TRY(cudaFuncSetAttribute(score_pass2_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024));
  if (dev < 64) done |= (uint64_t)1 << dev;
  return KVC_OK;
}

template <int D>
kvc_status launch_all(const CUtensorMap& kmap, ScoreArgs a, const Geometry& gm, int hp, cudaStream_t st) {
  const size_t smem = Smem<D>::total(a.Rq);
  kvc_status s = set_smem_attrs<D>(smem);
  if (s != KVC_OK) return s;
  const int grid_x = (int)((a.total + a.chunk_keys - 1) / a.chunk_keys) + a.B;
  for (int g0 = 0; g0 < a.Hkv; g0 += hp) {
    a.g0 = g0;
    dim3 grid(grid_x, std::min(hp, a.Hkv - g0));
    a.tmem_cols = gm.cols1;
    score_pass1_kernel<D><<<grid, kThreadsScore, smem, st>>>(kmap, a);
    KVC_CUDA_TRY(cudaGetLastError());
    a.tmem_cols = gm.cols2;
    score_pass2_kernel<D><<<grid, kThreadsScore, smem, st>>>(kmap, a);
    KVC_CUDA_TRY(cudaGetLastError());
    count_launch(2);
  }
  return KVC_OK;
}

kvc_status score_impl(const uint16_t* q, int64_t q_sb, int64_t q_sw, int64_t q_sh, const uint16_t* k,
                      int64_t k_sn, int64_t k_sh, const int32_t* cu, int B, int64_t total,
                      const kvc_score_params* p, float* scores, float* tsp, float* accum, void* ws,
                      size_t ws_bytes, int32_t* err, cudaStream_t st) {
  kvc_status s = check_params(p);
  if (s != KVC_OK) return s;
  KVC_CHECK_ARG(q && k && scores, "q_win, k and scores must be non-NULL");
  KVC_CHECK_ARG(aligned(q, 16) && aligned(k, 16), "q_win and k must be 16-byte aligned");
  KVC_CHECK_ARG(q_sw % 8 == 0 && q_sh % 8 == 0 && q_sb % 8 == 0 && q_sw >= 0 && q_sh >= 0 && q_sb >= 0,
                "q strides must be non-negative multiples of 8 elements");
  KVC_CHECK_ARG(k_sn % 8 == 0 && k_sh % 8 == 0 && k_sn > 0 && k_sh >= 0,
                "k strides must be positive multiples of 8 elements");
  KVC_CHECK_ARG(k_sn * 2 < (int64_t(1) << 40) && k_sh * 2 < (int64_t(1) << 40), "k strides too large");
  KVC_CHECK_ARG(aligned(scores, 16) && (!tsp || aligned(tsp, 16)) && (!accum || aligned(accum, 16)),
                "scores / tsp / accum must be 16-byte aligned");
  const size_t need = score_ws_bytes(p, B, total);
  if (!ws || ws_bytes < need || !aligned(ws, kWsAlign))
    return fail(KVC_ERR_WORKSPACE, "score workspace missing, too small or not 256-B aligned");
  if (total == 0) return KVC_OK;

  const Geometry gm = geometry(p);
  const int Hkv = p->num_kv_heads, d = p->head_dim;
  WsCursor wc{static_cast<char*>(ws), ws_bytes};
  wc.take<char>(kWsAlign);
  const int mc = max_chunks_bound(total, B);
  float* part_m = wc.take<float>((size_t)Hkv * mc * gm.Rq);
  double* part_l = wc.take<double>((size_t)Hkv * mc * gm.Rq);
  if (!wc.ok) return fail(KVC_ERR_WORKSPACE, "score workspace too small");

  auto encode = get_encode_fn();
  if (!encode) return fail(KVC_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  CUtensorMap kmap;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)Hkv, (cuuint64_t)total};
  cuuint64_t strides[2] = {(cuuint64_t)(k_sh * 2), (cuuint64_t)(k_sn * 2)};
  cuuint32_t box[3] = {64u, 1u, (cuuint32_t)kTile};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  if (Hkv == 1) strides[0] = (cuuint64_t)(k_sn * 2);  // a size-1 dim still needs a legal stride
  CUresult cr = encode(&kmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(k), dims, strides, box,
                       estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return fail(KVC_ERR_CUDA, "cuTensorMapEncodeTiled failed for K");

  // heads per launch: K of those heads should stay in L2 between the passes
  int dev = 0, l2 = 0;
  KVC_CUDA_TRY(cudaGetDevice(&dev));
  KVC_CUDA_TRY(cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev));
  const double head_bytes = (double)total * d * 2.0;
  int hp = (int)std::max(1.0, std::floor(0.6 * (double)l2 / head_bytes));
  hp = std::min(hp, Hkv);
  // chunk size: about one wave of CTAs per launch
  const int sms = num_sms();
  const int64_t tiles = (total + kTile - 1) / kTile + (B > 1 ? B : 0);
  const int64_t slots = std::max<int64_t>(1, sms / hp);
  const int64_t chunk_tiles = std::max<int64_t>(kMinChunkTiles, (tiles + slots - 1) / slots);

  ScoreArgs a{};
  a.q = q;
  a.q_sb = q_sb;
  a.q_sw = q_sw;
  a.q_sh = q_sh;
  a.cu = cu;
  a.n = total;
  a.B = B;
  a.Hkv = Hkv;
  a.G = gm.G;
  a.w = p->window;
  a.R = gm.R;
  a.Rq = gm.Rq;
  a.Rn = gm.Rn;
  a.nb1 = gm.nb1;
  a.acc_stride1 = gm.acc_stride1;
  a.acc_stride = gm.acc_stride;
  a.chunk_keys = (int)(chunk_tiles * kTile);
  a.max_chunks = mc;
  a.c = (float)((double)p->scale * kLog2e);
  a.part_m = part_m;
  a.part_l = part_l;
  a.scores = scores;
  a.accum = accum;
  a.total = total;
  a.err = err;
  s = (d == 128) ? launch_all<128>(kmap, a, gm, hp, st) : launch_all<64>(kmap, a, gm, hp, st);
  if (s != KVC_OK) return s;
  if (tsp) {
    const int threads = 256;
    const int64_t blocks = std::min<int64_t>((total + threads - 1) / threads, (int64_t)sms * 8);
    tsp_sum_kernel<<<(unsigned)blocks, threads, 0, st>>>(scores, Hkv, total, tsp);
    count_launch();
    KVC_CUDA_TRY(cudaGetLastError());
  }
  return KVC_OK;
}

}  // namespace
}  // namespace kvc

using namespace kvc;

extern "C" kvc_status kvc_score_workspace_size(const kvc_score_params* p, int32_t batch, int64_t total_tokens,
                                               size_t* bytes) {
  clear_error();
  kvc_status s = check_params(p);
  if (s != KVC_OK) return s;
  KVC_CHECK_ARG(bytes != nullptr, "bytes must be non-NULL");
  KVC_CHECK_ARG(batch >= 1 && total_tokens >= 0 && total_tokens < (int64_t(1) << 31), "bad batch / total");
  *bytes = score_ws_bytes(p, batch, total_tokens);
  return KVC_OK;
}

extern "C" kvc_status kvc_score(const uint16_t* q_win, int64_t q_stride_w, int64_t q_stride_h, const uint16_t* k,
                                int64_t k_stride_n, int64_t k_stride_h, int64_t n, const kvc_score_params* p,
                                float* scores, float* tsp, float* accum, void* ws, size_t ws_bytes,
                                int32_t* dev_err, void* stream) {
  clear_error();
  kvc_status s = check_params(p);
  if (s != KVC_OK) return s;
  KVC_CHECK_ARG(n >= p->window && n < (int64_t(1) << 31), "need window <= n < 2^31");
  return score_impl(q_win, 0, q_stride_w, q_stride_h, k, k_stride_n, k_stride_h, nullptr, 1, n, p, scores, tsp,
                    accum, ws, ws_bytes, dev_err, (cudaStream_t)stream);
}

extern "C" kvc_status kvc_score_varlen(const uint16_t* q_win, int64_t q_stride_b, int64_t q_stride_w,
                                       int64_t q_stride_h, const uint16_t* k, int64_t k_stride_n,
                                       int64_t k_stride_h, const int32_t* cu_seqlens, int32_t batch, int64_t total,
                                       int64_t max_seqlen, const kvc_score_params* p, float* scores, float* tsp,
                                       float* accum, void* ws, size_t ws_bytes, int32_t* dev_err, void* stream) {
  clear_error();
  kvc_status s = check_params(p);
  if (s != KVC_OK) return s;
  KVC_CHECK_ARG(cu_seqlens != nullptr, "cu_seqlens must be non-NULL");
  KVC_CHECK_ARG(batch >= 1 && batch <= 1024, "batch must be in 1..1024");
  KVC_CHECK_ARG(total >= 0 && total < (int64_t(1) << 31), "total out of range");
  KVC_CHECK_ARG(max_seqlen >= 0, "max_seqlen must be >= 0");
  return score_impl(q_win, q_stride_b, q_stride_w, q_stride_h, k, k_stride_n, k_stride_h, cu_seqlens, batch,
                    total, p, scores, tsp, accum, ws, ws_bytes, dev_err, (cudaStream_t)stream);
}

// --------------------------------------------------------------------------
// Scoring with library-owned scratch, for callers that cannot allocate.
// --------------------------------------------------------------------------
// Some callers have no way to hand the library a workspace: an operator
// running inside another runtime's plugin interface that offers no scratch
// buffer, or a serving loop that must never call cudaMalloc once it is up
// (cudaMalloc can synchronise the device and stall every other stream).
// For them the chunk partials live in this file-scope device array instead
// of a caller buffer.  It is allocated when the library's module is loaded
// and every GPU that loads the library keeps its copy until the process
// exits.
namespace kvc {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[KVC_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device.  Host code may
// not use the symbol itself (it names a host-side shadow, not device
// memory), so the address is looked up once per device with that device
// current and cached.
kvc_status noalloc_scratch_ptr(void** out) {
  static std::mutex mu;
  static void* cache[64] = {};
  int dev = 0;
  KVC_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(KVC_ERR_UNSUPPORTED, "device ordinal >= 64");
  std::lock_guard<std::mutex> lk(mu);
  if (cache[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_noalloc_scratch)");
    cache[dev] = p;
  }
  *out = cache[dev];
  return KVC_OK;
}

}  // namespace
}  // namespace kvc

extern "C" kvc_status kvc_score_noalloc(const uint16_t* q_win, int64_t q_stride_w, int64_t q_stride_h,
                                        const uint16_t* k, int64_t k_stride_n, int64_t k_stride_h, int64_t n,
                                        const kvc_score_params* p, float* scores, float* tsp, float* accum,
                                        int32_t* dev_err, void* stream) {
  clear_error();
  kvc_status s = check_params(p);
  if (s != KVC_OK) return s;
  KVC_CHECK_ARG(n >= p->window && n < (int64_t(1) << 31), "need window <= n < 2^31");
  const size_t need = score_ws_bytes(p, 1, n);
  if (need > (size_t)KVC_NOALLOC_SCRATCH_BYTES)
    return fail(KVC_ERR_WORKSPACE, "kvc_score_noalloc needs " + std::to_string(need) +
                                       " bytes of scratch; its static scratch holds " +
                                       std::to_string((size_t)KVC_NOALLOC_SCRATCH_BYTES) +
                                       " (use kvc_score with a workspace)");
  void* ws = nullptr;
  s = noalloc_scratch_ptr(&ws);
  if (s != KVC_OK) return s;
  return score_impl(q_win, 0, q_stride_w, q_stride_h, k, k_stride_n, k_stride_h, nullptr, 1, n, p, scores, tsp,
                    accum, ws, (size_t)KVC_NOALLOC_SCRATCH_BYTES, dev_err, (cudaStream_t)stream);
}
