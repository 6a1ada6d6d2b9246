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
// multi-stage shared-memory ring.  One launch per pass covers every KV head,
// so the CTAs of a key range read whole token rows of K together (HBM
// streams best that way); pass 2 walks each chunk backwards, starting on the
// tiles pass 1 read last, which are still in L2.
//
// Warp roles per CTA: warp 0 issues TMA, warp 1 allocates TMEM and issues
// MMAs, the rest drain TMEM (epilogue: one group of four warps, one warp per
// TMEM lane quarter, for each accumulator buffer -- four buffers of 128
// columns in the common case, fewer when the accumulator is wider; the groups
// take the tiles in turn, so up to four warps per SM sub-partition hide each
// other's TMEM-load and MUFU latencies).  Every wait is bounded; on a timeout
// the CTA records KVC_DEV_ERR_TIMEOUT, lets in-flight copies and MMAs land,
// frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include <cuda_bf16.h>

#include "common.cuh"
#include "tc.cuh"

namespace kvc {
namespace {

constexpr int kTile = 128;       // keys per tile
constexpr int kMaxStages = 8;    // TMA ring depth bound (the host picks what fits)
constexpr int kMaxBufs = 4;      // TMEM accumulator buffers
constexpr int kCols = 32;        // accumulator columns per TMEM load
constexpr int kMinChunkTiles = 4;
constexpr int kBarEpi = 1;       // named barrier of all epilogue warps
constexpr double kLog2e = 1.4426950408889634;

// Block layout of both passes: warp 0 TMA producer, warp 1 MMA issuer, then
// one epilogue group of four warps (one per TMEM lane quarter) for each of the
// NB accumulator buffers.  Group i drains buffer i, i.e. tiles i, i + NB, ...
// Four groups hide each other's TMEM-load and exponential latencies; with
// fewer buffers (wide accumulators) a group per buffer beats groups that share
// one.
template <int NB>
struct Epi {
  static constexpr int kThreads = 128 * NB;
  static constexpr int kBlock = 64 + kThreads;
};

struct ScoreArgs {
  const uint16_t* q;
  int64_t q_sb, q_sw, q_sh;  // Q_win strides (elements): sequence, window row, head
  const int32_t* cu;         // nullptr: one sequence of n tokens
  int64_t n;                 // single-sequence length (ignored with cu)
  int B;
  int Hkv, G, w, R, Rq, Rn;  // rows per KV head, rows in smem, MMA N (pass 2)
  int nb1;                   // 128-row blocks in pass 1
  int acc_stride;            // TMEM columns between accumulator buffers (this pass)
  int nbuf;                  // TMEM accumulator buffers = epilogue groups (this pass): 2, 3 or 4
  int stages;                // TMA ring depth
  int fold;                  // pass 2: the row bias rides in one extra MMA K-step
  float keep_frac;           // pass 1: trailing fraction of each chunk left at normal L2 priority
  uint32_t tmem_cols;        // TMEM columns allocated (this pass)
  int g0;                    // first KV head of this launch
  int chunk_keys;
  int max_chunks;            // partial slots per KV head
  float c;                   // scale * log2(e)
  float* part_m;             // [Hkv][max_chunks][Rq]: one row of partials per chunk
  double* part_l;            // [Hkv][max_chunks][Rq]
  uint2* qsplit;             // [B][Hkv][Rq]: -bias/c as three bf16 parts (words w0, w1)
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
// reverse: CTA 0 takes the last chunk (pass 2 walks the keys backwards, so
// it starts on what pass 1 left in L2).
__device__ __forceinline__ Work map_work(const ScoreArgs& a, int linear, bool reverse) {
  if (reverse) {
    int total = 0;
    for (int b = 0; b < a.B; ++b) {
      const SeqSpan s = seq_span(a.cu, b, a.n);
      const bool bad = s.start < 0 || s.len < a.w || s.start + s.len > a.total;
      total += bad ? 1 : (int)((s.len + a.chunk_keys - 1) / a.chunk_keys);
    }
    if (linear >= total) return Work{0, 0, 0, 0, 0, 0, false, false};
    linear = total - 1 - linear;
  }
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

struct Barriers {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t tfull[kMaxBufs];
  uint64_t tempty[kMaxBufs];
  uint64_t bias_ready;  // pass 2: the epilogue wrote the bias block
  uint32_t tmem_base;
  int abort;
};

// Shared memory: [Q rows, swizzled][pass 2: ones | bias block][K stage ring]
// [barriers].  The pass-2 blocks hold one extra K-step of the MMA: a
// [128 keys x 16] block of (1, 1, 1, 0, ...) and a [Rq x 16] block of each
// row's (h1, h2, h3, 0, ...) with h1 + h2 + h3 = -bias / c (three bf16 parts
// of an fp32-accurate value), 32-byte rows with the 32-byte swizzle.  Pass 1
// exchanges its group partials through the K ring once every tile is done.
template <int D>
struct Smem {
  static constexpr int kChunks = D / 64;  // 64-element (128 B) swizzle columns
  static constexpr int kStageBytes = kChunks * kTile * 128;
  static constexpr size_t kOnesBytes = (size_t)kTile * 32;
  static constexpr size_t kTail = 512;  // barriers
  static constexpr size_t kExchangeBytes = (size_t)(kMaxBufs - 1) * 256 * (4 + 8);
  static_assert(kExchangeBytes <= (size_t)kStageBytes * 2, "pass-1 exchange must fit in two stages");
  __host__ __device__ static size_t q_bytes(int Rq) { return (size_t)kChunks * Rq * 128; }
  __host__ __device__ static size_t fold_bytes(int Rq, int fold) { return fold ? kOnesBytes + (size_t)Rq * 32 : 0; }
  __host__ __device__ static size_t total(int Rq, int stages, int fold) {
    return 1024 /*alignment slack*/ + q_bytes(Rq) + fold_bytes(Rq, fold) + (size_t)stages * kStageBytes + kTail;
  }
};

template <int D>
struct SmemPtrs {
  uint8_t* qs;
  uint8_t* ones;  // pass 2 only
  uint8_t* qb;    // pass 2 only
  uint8_t* kst;
  Barriers* bars;
  float* ex_m;   // [groups - 1][256], in the K ring (pass 1, after the last tile)
  double* ex_l;  // [groups - 1][256]
  __device__ SmemPtrs(uint8_t* raw, const ScoreArgs& a) {
    uint8_t* s = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    qs = s;
    ones = qs + Smem<D>::q_bytes(a.Rq);
    qb = ones + Smem<D>::kOnesBytes;
    kst = qs + Smem<D>::q_bytes(a.Rq) + Smem<D>::fold_bytes(a.Rq, a.fold);
    bars = reinterpret_cast<Barriers*>(kst + (size_t)a.stages * Smem<D>::kStageBytes);
    ex_m = reinterpret_cast<float*>(kst);
    ex_l = reinterpret_cast<double*>(ex_m + (kMaxBufs - 1) * 256);
  }
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

// Barrier init (one thread) for the stage ring and the TMEM buffers.  Each
// use of a buffer is drained by the four warps of its epilogue group.
__device__ __forceinline__ void init_barriers(Barriers* bars, int stages, int nbuf, int epi_threads) {
  for (int s = 0; s < stages; ++s) {
    tc::mbar_init(&bars->full[s], 1);
    tc::mbar_init(&bars->empty[s], 1);
  }
  for (int s = 0; s < nbuf; ++s) {
    tc::mbar_init(&bars->tfull[s], 1);
    tc::mbar_init(&bars->tempty[s], 4);
  }
  tc::mbar_init(&bars->bias_ready, epi_threads);
  bars->abort = 0;
  tc::fence_mbar_init();
}

// Producer: stream the chunk's K tiles of head g into the stage ring.
//
// L2 policy: K is read by both passes, and more of it than L2 holds.  Pass 1
// loads the leading part of each chunk evict_first and its trailing
// `keep_frac` at normal priority; pass 2 walks the chunk backwards, so it
// starts on those trailing tiles while they are still in L2, and loads
// everything evict_first (nothing reads K after it).
template <int D>
__device__ __forceinline__ void produce(const void* kmap, Barriers* bars, uint8_t* kst, int stages, int g,
                                        int64_t row0, int ntiles, bool reverse, float keep_frac) {
  constexpr int kChunks = D / 64;
  constexpr uint32_t kBytes = (uint32_t)Smem<D>::kStageBytes;
  const uint64_t pol_first = tc::l2_policy_evict_first();
  const uint64_t pol_keep = tc::l2_policy_evict_normal();
  const int first_kept = reverse ? ntiles : ntiles - (int)((float)ntiles * keep_frac);
  int issued = 0;
  for (int t = 0; t < ntiles; ++t) {
    const int s = t % stages;
    const int u = t / stages;
    if (u > 0 && !tc::mbar_wait(&bars->empty[s], (u - 1) & 1, &bars->abort)) break;
    tc::mbar_arrive_expect_tx(&bars->full[s], kBytes);
    uint8_t* dst = kst + (size_t)s * Smem<D>::kStageBytes;
#pragma unroll
    for (int c = 0; c < kChunks; ++c)
      tc::tma_load_3d_hint(dst + c * kTile * 128, kmap, &bars->full[s], c * 64, g,
                           (int)(row0 + (int64_t)(reverse ? ntiles - 1 - t : t) * kTile),
                           t >= first_kept ? pol_keep : pol_first);
    issued = t + 1;
  }
  if (bars->abort) {
    // let every copy already issued land before the CTA can exit
    for (int t = std::max(0, issued - stages); t < issued; ++t)
      tc::mbar_drain(&bars->full[t % stages], (t / stages) & 1);
  }
}

// MMA issuer (one thread).  kRowsOnM: pass 1 (A = Q rows, B = K tile);
// otherwise pass 2 (A = K tile, B = Q rows, N = Rn).
template <int D, bool kRowsOnM>
__device__ __forceinline__ void issue_mmas(const ScoreArgs& a, Barriers* bars, uint32_t tmem, uint8_t* qs,
                                           uint8_t* kst, uint8_t* ones, uint8_t* qb, int ntiles) {
  constexpr int kChunks = D / 64;
  const uint32_t idesc = kRowsOnM ? tc::idesc_bf16_f32(128, kTile) : tc::idesc_bf16_f32(128, a.Rn);
  // Shared-memory descriptors are formed once: an MMA K-step or a stage only
  // moves the start-address field (bits [0,14): address >> 4; shared memory
  // is below 256 KB, so adding offset >> 4 never carries out of the field).
  // The issuing thread shares its sub-partition with busy epilogue warps, so
  // its instruction count per tile is kept small.
  const uint64_t q_desc0 = tc::desc_k_sw128(tc::smem_u32(qs));
  const uint64_t k_desc0 = tc::desc_k_sw128(tc::smem_u32(kst));
  const uint64_t ones_desc = tc::desc_k_sw32(tc::smem_u32(ones));
  const uint64_t qb_desc = tc::desc_k_sw32(tc::smem_u32(qb));
  const uint32_t q_chunk = (uint32_t)a.Rq * 8u;                          // (Rq * 128 B) >> 4
  constexpr uint32_t kChunk = (uint32_t)(kTile * 128) >> 4;                 // one 64-column block of a K tile
  constexpr uint32_t kStage = (uint32_t)Smem<D>::kStageBytes >> 4;
  int issued = 0;
  const bool go = kRowsOnM || tc::mbar_wait(&bars->bias_ready, 0, &bars->abort);
  for (int t = 0; go && t < ntiles; ++t) {
    const int s = t % a.stages;
    const int buf = t % a.nbuf, ub = t / a.nbuf;
    if (!tc::mbar_wait(&bars->full[s], (t / a.stages) & 1, &bars->abort)) break;
    if (ub > 0 && !tc::mbar_wait(&bars->tempty[buf], (ub - 1) & 1, &bars->abort)) break;
    tc::tc_fence_after();
    const uint64_t kd = k_desc0 + (uint64_t)((uint32_t)s * kStage);
    const int nblk = kRowsOnM ? a.nb1 : 1;
    for (int mb = 0; mb < nblk; ++mb) {
      const uint32_t d = tmem + (uint32_t)(buf * a.acc_stride + mb * kTile);
      const uint64_t qd = q_desc0 + (uint64_t)((uint32_t)mb * kChunk);  // row block mb of Q (pass 1)
#pragma unroll
      for (int c = 0; c < kChunks; ++c)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t qo = qd + (uint64_t)((uint32_t)c * q_chunk + (uint32_t)(ks * 2));
          const uint64_t ko = kd + (uint64_t)((uint32_t)c * kChunk + (uint32_t)(ks * 2));
          if (kRowsOnM)
            tc::mma_bf16(d, qo, ko, idesc, (c | ks) != 0);
          else
            tc::mma_bf16(d, ko, qo, idesc, (c | ks) != 0);
        }
      // pass 2: + (h1 + h2 + h3) = -bias/c on every (key, row)
      if (!kRowsOnM) tc::mma_bf16(d, ones_desc, qb_desc, idesc, 1u);
    }
    tc::mma_commit(&bars->empty[s]);
    tc::mma_commit(&bars->tfull[buf]);
    issued = t + 1;
  }
  if (issued > 0)  // the last MMAs landed before TMEM can be freed
    tc::mbar_drain(&bars->tfull[(issued - 1) % a.nbuf], ((issued - 1) / a.nbuf) & 1);
}

__device__ __forceinline__ void record_timeout(int32_t* err) { set_dev_err(err, KVC_DEV_ERR_TIMEOUT); }

// Epilogue warp, at tile t of its group: wait until the tile's accumulator is
// filled.  An mbarrier wait tells phases apart by parity only, so a waiter
// must never be two phases away from the barrier.  Every group owns one
// buffer: the buffer's previous use (tile t - nbuf) was this group's own
// previous tile, filled before and released by this warp, and the MMA cannot
// refill the buffer again before the group releases tile t -- so the fill
// barrier is exactly one phase behind this use.
__device__ __forceinline__ bool wait_filled(const ScoreArgs& a, Barriers* bars, int t) {
  return tc::mbar_wait(&bars->tfull[t % a.nbuf], (t / a.nbuf) & 1, &bars->abort);
}

// Online merge of (m, l) pairs in the log2 domain: l * 2^(m - M) summed.
__device__ __forceinline__ void merge_ml(float& M, double& L, float m2, double l2) {
  if (m2 == -INFINITY) return;
  if (M == -INFINITY) {
    M = m2;
    L = l2;
    return;
  }
  const float Mn = fmaxf(M, m2);
  L = L * (double)exp2f(M - Mn) + l2 * (double)exp2f(m2 - Mn);
  M = Mn;
}


// Load `ncol` (16 or 32) fp32 columns of this warp's 32 TMEM lanes starting
// at taddr into x[0..ncol).  Completion: KVC_TMEM_WAIT_LD32(x).
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&x)[kCols], int ncol) {
  if (ncol == 32) {
    KVC_TMEM_LD32(taddr, x);
  } else {
    KVC_TMEM_LD16(taddr, x);
  }
}

// Walk columns [0, ncols) of this warp's 32 lanes of one accumulator in
// groups of kCols: the next group's TMEM load is in flight while the current
// one is processed (proc(gi, x)); release() runs as soon as the last load has
// landed, so the MMA may refill the buffer during the last group's math.
// The TMEM loads and waits are warp-collective (.sync.aligned): the warp is
// reconverged before the first one, and, when proc() branches or returns per
// lane (kDiverges), after every proc() call -- the one point every lane of the
// warp always reaches.
template <bool kDiverges, class Proc, class Release>
__device__ __forceinline__ void walk_columns(uint32_t base, int ncols, Proc&& proc, Release&& release) {
  uint32_t xa[kCols], xb[kCols];
  const int ng = (ncols + kCols - 1) / kCols;
  __syncwarp();
  if (ng <= 0) {  // nothing to read (a warp whose rows are all padding): release at once
    release();
    return;
  }
  tmem_ld_cols(base, xa, min(kCols, ncols));
  for (int gi = 0; gi < ng; gi += 2) {
    KVC_TMEM_WAIT_LD32(xa);
    if (gi + 1 < ng)
      tmem_ld_cols(base + (uint32_t)((gi + 1) * kCols), xb, min(kCols, ncols - (gi + 1) * kCols));
    else
      release();
    proc(gi, xa);
    if (kDiverges) __syncwarp();
    if (gi + 1 < ng) {
      KVC_TMEM_WAIT_LD32(xb);
      if (gi + 2 < ng)
        tmem_ld_cols(base + (uint32_t)((gi + 2) * kCols), xa, min(kCols, ncols - (gi + 2) * kCols));
      else
        release();
      proc(gi + 1, xb);
      if (kDiverges) __syncwarp();
    }
  }
}

// Two consecutive accumulator values as a packed pair.
__device__ __forceinline__ float2 pair(const uint32_t (&x)[kCols], int e) {
  return make_float2(__uint_as_float(x[e]), __uint_as_float(x[e + 1]));
}

// acc += 2^(x[e]*c + off) over kCols values: per pair of columns one packed
// fma for the arguments, two ex2 and one packed add (four packed
// accumulators, i.e. eight independent sums).
__device__ __forceinline__ void acc_ex2(const uint32_t (&x)[kCols], float2 c2, float2 off2, float2 (&acc)[4]) {
#pragma unroll
  for (int e = 0; e < kCols; e += 2) {
    const float2 t = tc::fma2(pair(x, e), c2, off2);
    acc[(e >> 1) & 3] = tc::add2(acc[(e >> 1) & 3], make_float2(tc::ex2_approx(t.x), tc::ex2_approx(t.y)));
  }
}
__device__ __forceinline__ float sum4(const float2 (&acc)[4]) {
  const float2 u = tc::add2(tc::add2(acc[0], acc[1]), tc::add2(acc[2], acc[3]));
  return u.x + u.y;
}

// sum_e 2^(x[e]*c + off) over kCols values
__device__ __forceinline__ float sum_ex2(const uint32_t (&x)[kCols], float c, float off) {
  float2 acc[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) acc[u] = make_float2(0.f, 0.f);
  acc_ex2(x, make_float2(c, c), make_float2(off, off), acc);
  return sum4(acc);
}

__device__ __forceinline__ float max_cols(const uint32_t (&x)[kCols]) {
  float m8[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) m8[u] = -INFINITY;
#pragma unroll
  for (int e = 0; e < kCols; ++e) m8[e & 7] = fmaxf(m8[e & 7], __uint_as_float(x[e]));
  return fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
}

// Pass-1 update of one row with kCols logits (raw dot products) of consecutive
// keys.  The exponentials use the row's running reference `ref` (log2
// domain) instead of a fresh per-tile max: only when that would overflow the
// fp32 partial sum (a logit more than ~94 above the reference) -- and on the
// first values a row sees, when ref is -inf -- is the exact max taken and the
// running sum rescaled.
__device__ __forceinline__ void pass1_group(uint32_t (&x)[kCols], float c, float& ref, double& l) {
  float s = sum_ex2(x, c, -ref);
  if (!(s < 0x1p100f)) {  // overflow, or NaN from ref = -inf (a per-thread branch)
    const float hmax = max_cols(x);
    if (hmax == -INFINITY) return;  // every key masked
    const float nr = fmaxf(ref, hmax * c);
    if (ref != -INFINITY) l *= (double)exp2f(ref - nr);
    ref = nr;
    s = sum_ex2(x, c, -ref);
  }
  l += (double)s;
}

// --------------------------------------------------------------------------
// pass 1: per-row max / sum over a chunk of keys
// --------------------------------------------------------------------------
template <int D, int NB>
__global__ void __launch_bounds__(Epi<NB>::kBlock, 1)
score_pass1_kernel(const __grid_constant__ CUtensorMap kmap, const ScoreArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  const SmemPtrs<D> sp(smem_raw, a);
  Barriers* bars = sp.bars;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = a.g0 + blockIdx.y;
  const Work wk = map_work(a, blockIdx.x, false);
  if (!wk.valid) return;
  if (wk.bad) {
    if (threadIdx.x == 0 && blockIdx.y == 0) set_dev_err(a.err, KVC_DEV_ERR_SEQLENS);
    return;
  }
  const int64_t k0 = (int64_t)wk.chunk * a.chunk_keys;
  const int64_t k1 = std::min<int64_t>(wk.len, k0 + a.chunk_keys);
  const int ntiles = (int)((k1 - k0 + kTile - 1) / kTile);

  if (threadIdx.x == 0) init_barriers(bars, a.stages, a.nbuf, Epi<NB>::kThreads);
  if (warp == 0 && lane == 0) tc::prefetch_tmap(&kmap);
  if (warp == 1) {
    tc::tmem_alloc(&bars->tmem_base, a.tmem_cols);
    tc::tmem_relinquish();
  }
  load_q_swizzled<D>(a, wk.b, g, sp.qs);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0) produce<D>(&kmap, bars, sp.kst, a.stages, g, wk.start + k0, ntiles, false, a.keep_frac);
  } else if (warp == 1) {
    if (lane == 0) issue_mmas<D, true>(a, bars, tmem, sp.qs, sp.kst, sp.ones, sp.qb, ntiles);
  } else {
    // ---- epilogue: one row per thread and row block; the groups take the
    // tiles in turn.  A tile is nb1 row blocks x 128 key columns.
    const int grp = (warp - 2) >> 2;
    const int q = warp & 3;         // TMEM lane quarter of this warp
    const int rl = 32 * q + lane;  // lane within a 128-row block
    constexpr int kPerBlock = kTile / kCols;
    float m_run[2] = {-INFINITY, -INFINITY};
    double l_run[2] = {0.0, 0.0};
    const int64_t first_window_key = wk.len - a.w;  // earliest window row sees keys <= this
    // row blocks in which this warp owns window rows: a warp whose 32 rows of a
    // block are all padding skips that block's columns
    const int blocks_w = std::min(a.nb1, std::max(0, (a.R - 32 * q + kTile - 1) / kTile));
    for (int t = grp; t < ntiles; t += NB) {
      const int buf = t % a.nbuf;
      if (!wait_filled(a, bars, t)) break;
      tc::tc_fence_after();
      const int64_t j0 = k0 + (int64_t)t * kTile;  // first key of the tile (sequence-local)
      const bool masked = (j0 + kTile - 1 > first_window_key);
      // every lane of a walked block is a window row and no key is masked
      const bool fast = !masked && (a.R % 32) == 0;
      const uint32_t base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * a.acc_stride);
      walk_columns<true>(
          base, blocks_w * kTile,
          [&](int gi, uint32_t(&x)[kCols]) {
            if (fast) {  // warp-uniform: the common case
              if (gi < kPerBlock)
                pass1_group(x, a.c, m_run[0], l_run[0]);
              else
                pass1_group(x, a.c, m_run[1], l_run[1]);
              return;
            }
            const int mb = gi / kPerBlock;
            const int r = mb * kTile + rl;
            if (r >= a.R) return;
            if (masked) {
              // keys past this row's own position (or past the sequence) get -inf
              const int64_t lim = first_window_key + r / a.G - (j0 + (gi % kPerBlock) * kCols);
#pragma unroll
              for (int e = 0; e < kCols; ++e)
                if (e > lim) x[e] = __float_as_uint(-INFINITY);
            }
            if (mb == 0)
              pass1_group(x, a.c, m_run[0], l_run[0]);
            else
              pass1_group(x, a.c, m_run[1], l_run[1]);
          },
          [&]() {
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->tempty[buf]);
          });
    }
    // ---- merge the groups, then one chunk partial per row (combined later)
    tc::named_bar_sync(kBarEpi, Epi<NB>::kThreads);
    if (grp > 0) {
#pragma unroll
      for (int mb = 0; mb < 2; ++mb) {
        if (mb >= a.nb1) break;
        sp.ex_m[(grp - 1) * 256 + mb * kTile + rl] = m_run[mb];
        sp.ex_l[(grp - 1) * 256 + mb * kTile + rl] = l_run[mb];
      }
    }
    tc::named_bar_sync(kBarEpi, Epi<NB>::kThreads);
    if (grp == 0 && !bars->abort) {
#pragma unroll
      for (int mb = 0; mb < 2; ++mb) {
        if (mb >= a.nb1) break;
        const int r = mb * kTile + rl;
        if (r >= a.R) continue;
        float M = m_run[mb];
        double L = l_run[mb];
        for (int o = 0; o < NB - 1; ++o) merge_ml(M, L, sp.ex_m[o * 256 + mb * kTile + rl], sp.ex_l[o * 256 + mb * kTile + rl]);
        const size_t slot = ((size_t)g * a.max_chunks + wk.gid) * a.Rq + r;
        a.part_m[slot] = M;
        a.part_l[slot] = L;
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

// -bias / c as three bf16 parts (words w0 = h1 | h2 << 16, w1 = h3) whose fp32
// sum is accurate to ~2^-26 relative: each part holds the rounding residual
// of the previous one.
__device__ __forceinline__ uint2 split_bias3(double v) {
  const __nv_bfloat16 h1 = __float2bfloat16_rn((float)v);
  const double r1 = v - (double)__bfloat162float(h1);
  const __nv_bfloat16 h2 = __float2bfloat16_rn((float)r1);
  const double r2 = r1 - (double)__bfloat162float(h2);
  const __nv_bfloat16 h3 = __float2bfloat16_rn((float)r2);
  return make_uint2((uint32_t)__bfloat16_as_ushort(h1) | ((uint32_t)__bfloat16_as_ushort(h2) << 16),
                    (uint32_t)__bfloat16_as_ushort(h3));
}
constexpr uint32_t kPadBias = 0xFF7Fu;  // padded row: -3.39e38, so 2^(x * c) = 0

// --------------------------------------------------------------------------
// between the passes: per (sequence, KV head, row) combine the chunk partials
// into the row's bias b_r = M + log2(sum_c l_c 2^(m_c - M)), M = max_c m_c,
// and store -b_r / c as three bf16 parts (their fp32 sum is accurate to
// ~2^-26 relative; each part holds the rounding residual of the previous
// one).  Pass 2 multiplies them by ones in one extra MMA K-step.
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(256) score_combine_kernel(const ScoreArgs a) {
  // pass 2 may launch once pass 1 is complete: its prologue (barriers, TMEM,
  // Q, first K tiles) then overlaps this kernel
  pdl_wait();
  pdl_trigger();
  const int g = blockIdx.x, b = blockIdx.y;
  int gid0 = 0, nch = 0;
  bool bad = false;
  for (int bb = 0; bb <= b; ++bb) {
    const SeqSpan sp = seq_span(a.cu, bb, a.n);
    const bool bd = sp.start < 0 || sp.len < a.w || sp.start + sp.len > a.total;
    const int n = bd ? 1 : (int)((sp.len + a.chunk_keys - 1) / a.chunk_keys);
    if (bb < b) {
      gid0 += n;
    } else {
      nch = n;
      bad = bd;
    }
  }
  if (bad) return;
  for (int r = threadIdx.x; r < a.Rn; r += blockDim.x) {
    uint2 bias = make_uint2(kPadBias, 0u);
    if (r < a.R) {
      const float* pm = a.part_m + ((size_t)g * a.max_chunks + gid0) * a.Rq + r;
      const double* pl = a.part_l + ((size_t)g * a.max_chunks + gid0) * a.Rq + r;
      const size_t cs = (size_t)a.Rq;  // stride between consecutive chunks
      float M = -INFINITY;
      double L = 0.0;
      constexpr int kB = 16;
      for (int c0 = 0; c0 < nch; c0 += kB) {
        float mv[kB];
        double lv[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          const bool in = c0 + u < nch;
          mv[u] = in ? pm[(c0 + u) * cs] : -INFINITY;
          lv[u] = in ? pl[(c0 + u) * cs] : 0.0;
        }
        float bm = -INFINITY;
#pragma unroll
        for (int u = 0; u < kB; ++u) bm = fmaxf(bm, mv[u]);
        if (bm == -INFINITY) continue;
        const float Mn = fmaxf(M, bm);
        double acc = 0.0;
#pragma unroll
        for (int u = 0; u < kB; ++u)
          if (mv[u] != -INFINITY) acc += lv[u] * (double)exp2f(mv[u] - Mn);
        L = (M == -INFINITY) ? acc : L * (double)exp2f(M - Mn) + acc;
        M = Mn;
      }
      bias = split_bias3(-((double)M + log2(L)) / (double)a.c);
    }
    a.qsplit[((size_t)b * a.Hkv + g) * a.Rq + r] = bias;
  }
}

// With the rows' softmax normalisers given -- lse[i][h] = ln of the sum of
// exp(scale * q.k) over the keys window row i of query head h sees, the
// log-sum-exp a causal prefill attention returns for that query -- row
// r = i*G + h_local has b_r = lse * log2(e) in the log2 domain, and pass 2
// needs only -b_r / c = -lse / scale: pass 1 and the combine do not run.
// One sequence; grid = KV heads.
__global__ void __launch_bounds__(256) score_lse_bias_kernel(const ScoreArgs a, const float* __restrict__ lse,
                                                             int64_t ls_w, int64_t ls_h) {
  pdl_wait();  // an earlier kernel of the stream may still read the bias block
  pdl_trigger();
  const int g = blockIdx.x;
  for (int r = threadIdx.x; r < a.Rn; r += blockDim.x) {
    uint2 bias = make_uint2(kPadBias, 0u);
    if (r < a.R) {
      const int i = r / a.G, h = g * a.G + r % a.G;
      bias = split_bias3(-((double)lse[(int64_t)i * ls_w + (int64_t)h * ls_h] * kLog2e) / (double)a.c);
    }
    a.qsplit[(size_t)g * a.Rq + r] = bias;
  }
}

// --------------------------------------------------------------------------
// pass 2: per-key sum of normalised probabilities over the window rows
// --------------------------------------------------------------------------
template <int D, int NB>
__global__ void __launch_bounds__(Epi<NB>::kBlock, 1)
score_pass2_kernel(const __grid_constant__ CUtensorMap kmap, const ScoreArgs a) {
  // Before pdl_wait() this kernel reads only the call's inputs (Q, K, the
  // sequence offsets) and shared memory; the combined biases and every global
  // write come after it.  Its own dependents may launch only once it is
  // complete (no early trigger: a dependent resident early could hold the SM
  // a not yet scheduled CTA of this grid needs).
  extern __shared__ uint8_t smem_raw[];
  const SmemPtrs<D> sp(smem_raw, a);
  Barriers* bars = sp.bars;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = a.g0 + blockIdx.y;
  const Work wk = map_work(a, blockIdx.x, true);
  if (!wk.valid) return;
  if (wk.bad) {
    pdl_wait();
    // leave nothing stale behind: zero whatever part of the row is addressable
    if (wk.start >= 0 && wk.len > 0 && wk.start + wk.len <= a.total)
      for (int64_t j = threadIdx.x; j < wk.len; j += blockDim.x) a.scores[(int64_t)g * a.total + wk.start + j] = 0.f;
    return;
  }
  const int64_t k0 = (int64_t)wk.chunk * a.chunk_keys;
  const int64_t k1 = std::min<int64_t>(wk.len, k0 + a.chunk_keys);
  const int ntiles = (int)((k1 - k0 + kTile - 1) / kTile);

  if (threadIdx.x == 0) init_barriers(bars, a.stages, a.nbuf, Epi<NB>::kThreads);
  if (warp == 0 && lane == 0) tc::prefetch_tmap(&kmap);
  if (warp == 1) {
    tc::tmem_alloc(&bars->tmem_base, a.tmem_cols);
    tc::tmem_relinquish();
  }
  {
    // constant operands of the extra K-step: ones block (keys) and a zeroed
    // bias block (rows); row r's 16-byte chunk 0 sits at chunk (r >> 2) & 1
    uint4* ones4 = reinterpret_cast<uint4*>(sp.ones);
    for (int v = threadIdx.x; v < (int)(Smem<D>::kOnesBytes / 16); v += blockDim.x) {
      const int r = v >> 1, ch = v & 1;
      ones4[v] = (ch == ((r >> 2) & 1)) ? make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u) : make_uint4(0u, 0u, 0u, 0u);
    }
    uint4* qb4 = reinterpret_cast<uint4*>(sp.qb);
    for (int v = threadIdx.x; v < a.Rq * 2; v += blockDim.x) qb4[v] = make_uint4(0u, 0u, 0u, 0u);
  }
  load_q_swizzled<D>(a, wk.b, g, sp.qs);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0) produce<D>(&kmap, bars, sp.kst, a.stages, g, wk.start + k0, ntiles, true, a.keep_frac);
  } else if (warp == 1) {
    if (lane == 0) issue_mmas<D, false>(a, bars, tmem, sp.qs, sp.kst, sp.ones, sp.qb, ntiles);
  } else {
    // ---- epilogue prologue: this (sequence, head)'s bias rows into the bias
    // block of the extra MMA K-step, so the accumulator already holds
    // x - b_r / c.  TMA fills the pipeline meanwhile; the MMA waits for
    // bias_ready.
    {
      pdl_wait();  // the combined biases (previous kernel)
      const int r = threadIdx.x - 64;
      if (r < a.Rn) {
        const uint2 wv = a.qsplit[((size_t)wk.b * a.Hkv + g) * a.Rq + r];
        *reinterpret_cast<uint4*>(sp.qb + (size_t)r * 32 + (size_t)((r >> 2) & 1) * 16) = make_uint4(wv.x, wv.y, 0u, 0u);
      }
      tc::fence_proxy_async_smem();  // visible to the MMA's operand reads
      tc::mbar_arrive(&bars->bias_ready);
    }
    // ---- epilogue: one key per thread; the groups take the tiles in turn and
    // walk a tile's Rn row columns kCols at a time.
    const int grp = (warp - 2) >> 2;
    const int q = warp & 3;
    const int kl = 32 * q + lane;  // key within the tile
    const int64_t first_window_key = wk.len - a.w;
    for (int t = grp; t < ntiles; t += NB) {
      const int buf = t % a.nbuf;
      if (!wait_filled(a, bars, t)) break;
      tc::tc_fence_after();
      const int tp = ntiles - 1 - t;                    // tiles are walked backwards
      const int64_t j = k0 + (int64_t)tp * kTile + kl;  // this thread's key (sequence-local)
      const bool masked = (k0 + (int64_t)tp * kTile + kTile - 1 > first_window_key);
      // first row that sees key j: row r = i*G + h belongs to window query i,
      // which sees keys up to first_window_key + i
      const int64_t lim = j - first_window_key;
      const int rmin = lim <= 0 ? 0 : (int)std::min<int64_t>(lim * a.G, a.Rn);
      const uint32_t base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * a.acc_stride);
      float2 acc[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[u] = make_float2(0.f, 0.f);
      walk_columns<false>(
          base, a.Rn,
          [&](int gi, uint32_t(&x)[kCols]) {
            if (!masked && (a.Rn % kCols) == 0) {  // warp-uniform: the common case
              acc_ex2(x, make_float2(a.c, a.c), make_float2(0.f, 0.f), acc);
              return;
            }
            const int col0 = gi * kCols;
            const int ncol = min(kCols, a.Rn - col0);
            // columns past ncol (not loaded) and, on tiles reaching into the
            // window, keys past a row's own position get -inf, i.e. probability
            // 0.  Both are rare and warp-uniform, so they sit outside the math
            // loop, which stays branch-free and lets the exponentials interleave.
            if (ncol < kCols) {
#pragma unroll
              for (int e = 0; e < kCols; ++e)
                if (e >= ncol) x[e] = __float_as_uint(-INFINITY);
            }
            if (masked) {
#pragma unroll
              for (int e = 0; e < kCols; ++e)
                if (col0 + e < rmin) x[e] = __float_as_uint(-INFINITY);
            }
            acc_ex2(x, make_float2(a.c, a.c), make_float2(0.f, 0.f), acc);
          },
          [&]() {
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->tempty[buf]);
          });
      if (j < k1) {
        const float v = sum4(acc);
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
  pdl_wait();
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
  int G, R, Rq, Rn, nb1;
  int stride1, nbuf1;     // pass 1: TMEM columns per accumulator buffer, buffers
  int stride2, nbuf2;     // pass 2
  uint32_t cols1, cols2;  // TMEM columns allocated by pass 1 / pass 2
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
  // as many accumulator buffers (at most 4) as the 512 TMEM columns allow:
  // pass 1 4 or 2 (one or two 128-row blocks), pass 2 4, 3 or 2 (Rn <= 256)
  g.stride1 = g.nb1 * kTile;
  g.nbuf1 = std::min(kMaxBufs, 512 / g.stride1);
  g.stride2 = (g.Rn + 31) / 32 * 32;
  g.nbuf2 = std::min(kMaxBufs, 512 / g.stride2);
  g.cols1 = pow2_cols(g.nbuf1 * g.stride1);
  g.cols2 = pow2_cols(g.nbuf2 * g.stride2);
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
  s += round_up((size_t)B * p->num_kv_heads * gm.Rq * sizeof(uint2), kWsAlign);     // qsplit
  return s;
}

// The dynamic shared-memory limit is a per-device function attribute.
template <int D>
kvc_status set_smem_attrs(size_t bytes) {
  if (bytes > 227 * 1024) return fail(KVC_ERR_UNSUPPORTED, "score kernel shared memory above 227 KB");
  static ContextCache cache;
  return once_per_context(cache, [] {
    const void* fns[] = {(const void*)score_pass1_kernel<D, 2>, (const void*)score_pass1_kernel<D, 4>,
                         (const void*)score_pass2_kernel<D, 2>, (const void*)score_pass2_kernel<D, 3>,
                         (const void*)score_pass2_kernel<D, 4>};
    for (const void* f : fns)
      KVC_CUDA_TRY(cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024));
    return KVC_OK;
  });
}

// The window rows' log-sum-exp when the caller has it (one sequence), else none.
struct GivenLse {
  const float* p = nullptr;
  int64_t sw = 0, sh = 0;  // strides (elements) of window row and query head
};

template <int D>
kvc_status launch_all(const CUtensorMap& kmap, ScoreArgs a, const Geometry& gm, int hp, const GivenLse& lse,
                      cudaStream_t st) {
  // deepest TMA ring that fits next to the other blocks in 227 KB of shared memory
  const size_t budget = 227 * 1024;
  int stages[2];
  size_t smem[2];
  for (int pass = 0; pass < 2; ++pass) {
    const size_t fixed = Smem<D>::total(a.Rq, 0, pass);
    stages[pass] = fixed >= budget ? 0 : (int)std::min<size_t>(kMaxStages, (budget - fixed) / Smem<D>::kStageBytes);
    if (stages[pass] < 2) return fail(KVC_ERR_UNSUPPORTED, "score kernel: shared memory too small for 2 stages");
    smem[pass] = Smem<D>::total(a.Rq, stages[pass], pass);
  }
  // one epilogue group per buffer: only these block shapes are instantiated
  if ((gm.nbuf1 != 2 && gm.nbuf1 != 4) || gm.nbuf2 < 2 || gm.nbuf2 > 4)
    return fail(KVC_ERR_UNSUPPORTED, "score kernel: no block shape for this accumulator width");
  kvc_status s = set_smem_attrs<D>(std::max(smem[0], smem[1]));
  if (s != KVC_OK) return s;
  // chunks of all sequences: a bound (every sequence adds at most one partial
  // chunk); a single sequence needs exactly ceil(total / chunk)
  const int grid_x = (int)((a.total + a.chunk_keys - 1) / a.chunk_keys) + (a.cu ? a.B : 0);
  for (int g0 = 0; g0 < a.Hkv; g0 += hp) {
    a.g0 = g0;
    dim3 grid(grid_x, std::min(hp, a.Hkv - g0));
    a.acc_stride = gm.stride1;
    a.nbuf = gm.nbuf1;
    a.tmem_cols = gm.cols1;
    a.stages = stages[0];
    a.fold = 0;
    if (lse.p == nullptr) {
      {
        const Launch l(grid, dim3(64 + 128 * a.nbuf), smem[0], st);
        if (a.nbuf == 4)
          KVC_CUDA_TRY(l.run(score_pass1_kernel<D, 4>, kmap, a));
        else
          KVC_CUDA_TRY(l.run(score_pass1_kernel<D, 2>, kmap, a));
      }
      {
        const Launch l(dim3(a.Hkv, a.B), dim3(256), 0, st);
        KVC_CUDA_TRY(l.run(score_combine_kernel, a));
      }
      count_launch(2);
    } else {
      const Launch l(dim3(a.Hkv), dim3(256), 0, st);
      KVC_CUDA_TRY(l.run(score_lse_bias_kernel, a, lse.p, lse.sw, lse.sh));
      count_launch();
    }
    a.acc_stride = gm.stride2;
    a.nbuf = gm.nbuf2;
    a.tmem_cols = gm.cols2;
    a.stages = stages[1];
    a.fold = 1;
    {
      const Launch l(grid, dim3(64 + 128 * a.nbuf), smem[1], st);
      if (a.nbuf == 4)
        KVC_CUDA_TRY(l.run(score_pass2_kernel<D, 4>, kmap, a));
      else if (a.nbuf == 3)
        KVC_CUDA_TRY(l.run(score_pass2_kernel<D, 3>, kmap, a));
      else
        KVC_CUDA_TRY(l.run(score_pass2_kernel<D, 2>, kmap, a));
    }
    count_launch();
  }
  return KVC_OK;
}

kvc_status score_impl(const uint16_t* q, int64_t q_sb, int64_t q_sw, int64_t q_sh, const uint16_t* k,
                      int64_t k_sn, int64_t k_sh, const int32_t* cu, int B, int64_t total,
                      const kvc_score_params* p, float* scores, float* tsp, float* accum, void* ws,
                      size_t ws_bytes, int32_t* err, cudaStream_t st, const GivenLse& lse = GivenLse{}) {
  kvc_status s = check_params(p);
  if (s != KVC_OK) return s;
  KVC_CHECK_ARG(lse.p == nullptr || (cu == nullptr && B == 1), "a given log-sum-exp needs one sequence");
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
  uint2* qsplit = wc.take<uint2>((size_t)B * Hkv * gm.Rq);
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

  // all KV heads in one launch per pass: the CTAs of one key range read whole
  // [Hkv][d] token rows together, which keeps HBM streaming efficient (head
  // subsets per launch re-open every DRAM page once per subset)
  const int hp = Hkv;
  // trailing fraction of each chunk pass 1 leaves at normal L2 priority:
  // about 70 % of L2 worth of K (the rest of L2 serves everything else)
  int dev = 0, l2 = 0;
  KVC_CUDA_TRY(cudaGetDevice(&dev));
  KVC_CUDA_TRY(cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev));
  const double k_bytes = (double)total * Hkv * d * 2.0;
  const float keep_frac = (float)std::min(1.0, 0.7 * (double)l2 / k_bytes);
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
  a.chunk_keys = (int)(chunk_tiles * kTile);
  a.max_chunks = mc;
  a.c = (float)((double)p->scale * kLog2e);
  a.keep_frac = keep_frac;
  a.part_m = part_m;
  a.part_l = part_l;
  a.qsplit = qsplit;
  a.scores = scores;
  a.accum = accum;
  a.total = total;
  a.err = err;
  s = (d == 128) ? launch_all<128>(kmap, a, gm, hp, lse, st) : launch_all<64>(kmap, a, gm, hp, lse, st);
  if (s != KVC_OK) return s;
  if (tsp) {
    const int threads = 256;
    const int64_t blocks = std::min<int64_t>((total + threads - 1) / threads, (int64_t)sms * 8);
    const Launch l(dim3((unsigned)blocks), dim3(threads), 0, st);
    KVC_CUDA_TRY(l.run(tsp_sum_kernel, (const float*)scores, Hkv, total, tsp));
    count_launch();
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

extern "C" kvc_status kvc_score_lse(const uint16_t* q_win, int64_t q_stride_w, int64_t q_stride_h,
                                    const uint16_t* k, int64_t k_stride_n, int64_t k_stride_h, int64_t n,
                                    const kvc_score_params* p, const float* lse, int64_t lse_stride_w,
                                    int64_t lse_stride_h, float* scores, float* tsp, float* accum, void* ws,
                                    size_t ws_bytes, int32_t* dev_err, void* stream) {
  clear_error();
  kvc_status s = check_params(p);
  if (s != KVC_OK) return s;
  KVC_CHECK_ARG(n >= p->window && n < (int64_t(1) << 31), "need window <= n < 2^31");
  KVC_CHECK_ARG(lse != nullptr, "lse must be non-NULL");
  KVC_CHECK_ARG(lse_stride_w >= 0 && lse_stride_h >= 0, "lse strides must be >= 0");
  GivenLse given;
  given.p = lse;
  given.sw = lse_stride_w;
  given.sh = lse_stride_h;
  return score_impl(q_win, 0, q_stride_w, q_stride_h, k, k_stride_n, k_stride_h, nullptr, 1, n, p, scores, tsp,
                    accum, ws, ws_bytes, dev_err, (cudaStream_t)stream, given);
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
// memory), so the address is looked up with that device current and cached
// per device, keyed on the CUDA context: after a device reset the module is
// loaded again in a new context, the array may sit elsewhere, and the next
// call looks the address up afresh.
kvc_status noalloc_scratch_ptr(void** out) {
  static std::mutex mu;
  static void* ptr[64] = {};
  static uint64_t ctx[64] = {};
  int dev = 0;
  KVC_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(KVC_ERR_UNSUPPORTED, "device ordinal >= 64");
  std::lock_guard<std::mutex> lk(mu);
  const uint64_t id = current_context_id();
  if (ptr[dev] == nullptr || id == 0 || ctx[dev] != id) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_noalloc_scratch)");
    ptr[dev] = p;
    ctx[dev] = current_context_id();  // the lookup made the context current if it was not
  }
  *out = ptr[dev];
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
