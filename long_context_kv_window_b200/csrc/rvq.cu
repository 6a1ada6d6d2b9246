// rvq.cu -- residual vector quantisation of retained K/V rows on tcgen05.
//
// VQKV (gist.science 2603.16435) section 2: each cached vector is replaced by
// integer indices into codebooks; the quantisation is residual -- the first
// codebook encodes the vector, each later one the residual left by the
// stages before it.  Per stage s and row r (a whole head row of d values):
//     code_s = argmin_m ||r - C_s[m]||^2      (ties: the lowest index)
//     r     <- r - C_s[code_s]
//
// For 128 rows at a time the distances need r . C_s[m] for every codeword: a
// dense [128 x d] . [d x M] contraction, issued as tcgen05.mma kind::tf32
// (the residual is fp32, held in shared memory as the A operand; the stage's
// codebook is TMA-loaded beside it as the B operand; the scores land in
// TMEM).  tf32 keeps 10 mantissa bits, so the epilogue does not decide on the
// MMA's numbers alone: every codeword whose approximate score
//     a_m = ||C_s[m]||^2 - 2 r . C_s[m]        (||r||^2 is common to all m)
// is within the bound of the tf32 rounding of the best one is re-scored on the
// CUDA cores as the fp32 sum of (r_c - C_s[m]_c)^2, and the smallest of those
// (lowest index on ties) is the code -- the same decision as the definition,
// up to fp32 rounding of the distances.  The residual update is fp32.
//
// Thread 0 issues TMA and MMA; all 16 warps decide, four warps per row:
// the warp's TMEM lane quarter gives its 32 rows, and the four warps of a
// quarter take every fourth 16-codeword group of the scores and a quarter of
// the dimensions, exchanging per-row partials through shared memory (the
// decision of one row is a serial scan, so rows times column groups is the
// parallelism that hides its latencies).  Every wait is bounded; on a timeout
// the CTA records KVC_DEV_ERR_TIMEOUT, lets its copies and MMAs land, frees
// TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <mutex>

#include "common.cuh"
#include "tc.cuh"

namespace kvc {
namespace {

constexpr int kRows = 128;       // rows per CTA (MMA M)
constexpr int kRvqThreads = 512; // 16 warps, 4 per TMEM lane quarter (4 per SM sub-partition: 128 registers each)
constexpr int kColQ = 4;         // warps sharing one lane quarter (codeword groups / dimension quarters)
constexpr int kCandCap = 3072;   // (row, codeword) candidates a stage re-scores in parallel
constexpr int kBarAll = 5;       // named barrier of all 16 warps (1..4: one lane quarter's four)
constexpr int kMaxM = 256;       // codewords per codebook (MMA N <= 256)
constexpr int kMaxS = 16;        // stages

// tcgen05 instruction descriptor, kind::tf32: D fp32, A and B tf32, both K-major.
__host__ __device__ constexpr uint32_t idesc_tf32_f32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

struct RvqArgs {
  const uint16_t* x;  // [n][d] bf16, row stride x_stride
  int64_t x_stride;
  int64_t n;
  int S, M;
  int32_t* codes;     // [n][S]
  float* residual;    // [n][d] or nullptr
  int32_t* err;
};

struct RvqBars {
  uint64_t cb_full;   // codebook of the current stage landed
  uint64_t mma_done;  // scores of the current stage in TMEM
  uint32_t tmem_base;
  int abort;
  float cmax;         // max_m ||C_s[m]|| of the current stage
};

// Shared memory: [R: D/32 column blocks x 128 rows x 128 B][C: D/32 blocks x
// M rows x 128 B][cnorm[M]][barriers].  Both matrices are K-major with the
// 128-byte swizzle (32 fp32 per 128-byte row segment; 16-byte chunks XOR-ed
// with row & 7), which is what TMA writes for C and the MMA descriptors read.
template <int D>
struct RvqSmem {
  static constexpr int kBlocks = D / 32;
  static constexpr size_t kRBytes = (size_t)kBlocks * kRows * 128;
  static constexpr size_t kCBytes = (size_t)kBlocks * kMaxM * 128;
  static constexpr size_t kXBytes = (size_t)4 * kColQ * kRows * 4 + (size_t)kRows * 8 + (size_t)kCandCap * 4 + 16;
  static constexpr size_t kBytes = 1024 + kRBytes + kCBytes + kXBytes + kMaxM * 4 + 256;
};

// Per-row partials exchanged by the four warps of a lane quarter.
struct RvqExchange {
  float best[kColQ][kRows];  // approximate best score in the warp's codeword groups
  float rr[kColQ][kRows];    // ||r||^2 over the warp's quarter of the dimensions
  float dist[kColQ][kRows];  // (fallback path) exact best distance among the warp's candidates
  int arg[kColQ][kRows];     // (fallback path) its codeword (INT_MAX: none)
  unsigned long long key[kRows];  // exact best per row: fp32 distance bits << 32 | codeword
  uint32_t cand[kCandCap];   // candidates of the stage: row << 16 | codeword
  uint32_t ncand;            // candidates listed (may exceed kCandCap: then the fallback runs)
  uint32_t pad[3];
};
static_assert(sizeof(RvqExchange) == 4 * kColQ * kRows * 4 + kRows * 8 + kCandCap * 4 + 16, "exchange block");

// Byte offset of the 16-byte chunk holding elements c..c+3 (c % 4 == 0) of
// row `row` in a K-major SW128 matrix of `rows` rows.
__device__ __forceinline__ uint32_t sw_off(int row, int c, int rows) {
  const int blk = c >> 5, k16 = (c & 31) >> 2;
  return (uint32_t)(blk * rows * 128 + row * 128 + ((k16 ^ (row & 7)) << 4));
}

// Load two of this warp's 16-codeword score groups, cq + 4 k0 and cq + 4 (k0
// + 1), of its 32 TMEM lanes into x[0..15] and x[16..31], both in flight
// before one wait.  The group count is warp-uniform, so every load is
// executed by the whole warp.
__device__ __forceinline__ void load_group_pair(uint32_t base, int cq, int k0, int ngroups, uint32_t (&x)[32]) {
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int gi = cq + kColQ * (k0 + u);
    if (gi < ngroups) {
      uint32_t* xk = x + 16 * u;
      KVC_TMEM_LD16(base + (uint32_t)(16 * gi), xk);
    }
  }
  KVC_TMEM_WAIT_LD32(x);
}

template <int D>
__global__ void __launch_bounds__(kRvqThreads, 1)
rvq_encode_kernel(const __grid_constant__ CUtensorMap cmap, const RvqArgs a) {
  using L = RvqSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* R = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* C = R + L::kRBytes;
  RvqExchange* ex = reinterpret_cast<RvqExchange*>(C + L::kCBytes);
  float* cnorm = reinterpret_cast<float*>(C + L::kCBytes + L::kXBytes);
  RvqBars* bars = reinterpret_cast<RvqBars*>(cnorm + kMaxM);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t row0 = (int64_t)blockIdx.x * kRows;
  const int M = a.M;
  if (tid == 0) {
    tc::mbar_init(&bars->cb_full, 1);
    tc::mbar_init(&bars->mma_done, 1);
    ex->ncand = 0;
    bars->abort = 0;
    tc::fence_mbar_init();
    tc::prefetch_tmap(&cmap);
  }
  if (warp == 0) {
    tc::tmem_alloc(&bars->tmem_base, kMaxM);
    tc::tmem_relinquish();
  }
  pdl_wait();  // the rows may come from the previous kernel of the stream
  // rows -> fp32 residual (rows past n are zero); 16-byte loads of 8 bf16
  // where the row stride allows, else 4 x 2 bytes
  const bool vec = (a.x_stride % 8) == 0 && (reinterpret_cast<uintptr_t>(a.x) & 15) == 0;
  for (int i = tid; i < kRows * (D / 8); i += kRvqThreads) {
    const int row = i / (D / 8), c = (i % (D / 8)) * 8;
    float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
    if (row0 + row < a.n) {
      const uint16_t* src = a.x + (row0 + row) * a.x_stride + c;
      uint32_t w[4];
      if (vec) {
        const uint4 u = *reinterpret_cast<const uint4*>(src);
        w[0] = u.x; w[1] = u.y; w[2] = u.z; w[3] = u.w;
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) w[q] = (uint32_t)src[2 * q] | ((uint32_t)src[2 * q + 1] << 16);
      }
      v0 = make_float4(__uint_as_float(w[0] << 16), __uint_as_float(w[0] & 0xFFFF0000u),
                       __uint_as_float(w[1] << 16), __uint_as_float(w[1] & 0xFFFF0000u));
      v1 = make_float4(__uint_as_float(w[2] << 16), __uint_as_float(w[2] & 0xFFFF0000u),
                       __uint_as_float(w[3] << 16), __uint_as_float(w[3] & 0xFFFF0000u));
    }
    *reinterpret_cast<float4*>(R + sw_off(row, c, kRows)) = v0;
    *reinterpret_cast<float4*>(R + sw_off(row, c + 4, kRows)) = v1;
  }
  tc::fence_proxy_async_smem();  // residual visible to the MMA's operand reads
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  const int erow = 32 * (warp & 3) + lane;  // epilogue: TMEM lane quarter = warp % 4
  const int cq = warp >> 2;                 // which of the four warps of the quarter
  const bool has_row = row0 + erow < a.n;
  const uint32_t idesc = idesc_tf32_f32(kRows, M);
  int stage_done = 0;  // stages whose copies and MMAs have landed (thread 0's view)
  int cb_issued = 0, mma_issued = 0;  // thread 0: codebook copies / MMA batches issued

  for (int s = 0; s < a.S; ++s) {
    // the stage's candidate list and per-row bests start empty (every deciding
    // thread passes the barrier below before it touches them)
    if (warp == 0) {
      if (lane == 0) {
        ex->ncand = 0;
        bars->cmax = 0.f;
      }
      for (int i = lane; i < kRows; i += 32) ex->key[i] = ~0ull;
    }
    // ---- codebook of stage s -> C (TMA), then ||C_s[m]||^2 and max ||C_s[m]||
    if (tid == 0) {
      tc::mbar_arrive_expect_tx(&bars->cb_full, (uint32_t)(L::kBlocks * M * 128));
      for (int blk = 0; blk < L::kBlocks; ++blk)
        tc::tma_load_2d(C + (size_t)blk * M * 128, &cmap, &bars->cb_full, blk * 32, s * M);
      cb_issued = s + 1;
    }
    const bool got = tc::mbar_wait(&bars->cb_full, s & 1, &bars->abort);
    if (__syncthreads_or(!got)) break;
    // ---- scores: TMEM[row][m] = r . C_s[m] (tf32), 8 elements per K-step;
    // the codeword norms below are formed while the MMAs run
    if (tid == 0) {
      tc::tc_fence_after();
      const uint64_t ad = tc::desc_k_sw128(tc::smem_u32(R)), bd = tc::desc_k_sw128(tc::smem_u32(C));
#pragma unroll
      for (int k = 0; k < D / 8; ++k) {
        const uint32_t blk = (uint32_t)(k >> 2), kin = (uint32_t)((k & 3) * 32);
        tc::mma_tf32(tmem, ad + (uint64_t)((blk * kRows * 128 + kin) >> 4),
                          bd + (uint64_t)((blk * (uint32_t)M * 128 + kin) >> 4), idesc, k != 0);
      }
      tc::mma_commit(&bars->mma_done);
      mma_issued = s + 1;
    }
    float my_max = 0.f;
    for (int m = tid; m < M; m += kRvqThreads) {
      float acc = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; c += 4) {
        const float4 v = *reinterpret_cast<const float4*>(C + sw_off(m, c, M));
        acc = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, acc))));
      }
      cnorm[m] = acc;
      my_max = fmaxf(my_max, acc);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) my_max = fmaxf(my_max, __shfl_xor_sync(0xffffffffu, my_max, off));
    if (lane == 0) atomicMax(reinterpret_cast<int*>(&bars->cmax), __float_as_int(my_max));  // >= 0: int order
    const bool scored = tc::mbar_wait(&bars->mma_done, s & 1, &bars->abort);
    if (__syncthreads_or(!scored)) break;
    if (tid == 0) stage_done = s + 1;
    tc::tc_fence_after();
    const float cmax = sqrtf(bars->cmax);

    // ---- decision: approximate best, then exact fp32 distances of the candidates.
    // Warp (quarter q, part cq) scans the 16-codeword groups g = cq, cq + 4, ...
    // of its 32 rows and owns dimensions [cq D/4, (cq + 1) D/4) of them.
    {
      constexpr int kDq = D / kColQ;
      const int bar_id = 1 + (warp & 3);  // named barrier of the four warps of this lane quarter
      float rq = 0.f;
#pragma unroll
      for (int c = cq * kDq; c < (cq + 1) * kDq; c += 4) {
        const float4 v = *reinterpret_cast<const float4*>(R + sw_off(erow, c, kRows));
        rq = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, rq))));
      }
      const uint32_t base = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
      const int ngroups = M / 16;
      float best = INFINITY;
      // this warp's (up to four) 16-codeword groups, two loads in flight at a time
#pragma unroll
      for (int k0 = 0; k0 < kMaxM / 16 / kColQ; k0 += 2) {
        if (cq + kColQ * k0 >= ngroups) break;
        uint32_t x[32];
        load_group_pair(base, cq, k0, ngroups, x);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int gi = cq + kColQ * (k0 + u);
          if (gi < ngroups) {
#pragma unroll
            for (int e = 0; e < 16; ++e) best = fminf(best, cnorm[16 * gi + e] - 2.f * __uint_as_float(x[16 * u + e]));
          }
        }
      }
      ex->best[cq][erow] = best;
      ex->rr[cq][erow] = rq;
      tc::named_bar_sync(bar_id, 32 * kColQ);
      float rr = 0.f;
      best = INFINITY;
#pragma unroll
      for (int q = 0; q < kColQ; ++q) {
        rr += ex->rr[q][erow];
        best = fminf(best, ex->best[q][erow]);
      }
      // tf32 keeps 10 mantissa bits of each operand, so with the fp32 sums
      // |r.c - (MMA dot)| < 2^-8.9 ||r|| ||c|| and |||c||^2 - cnorm| < 2^-17
      // cmax^2 (d <= 128 terms).  Two approximate scores therefore differ from
      // the exact difference of the distances by less than
      // 2^-6.9 ||r|| cmax + 2^-16 cmax^2: every codeword within that band of
      // the best approximate score is a candidate, and the exact argmin is
      // always among them
      const float band = 0x1p-6f * sqrtf(rr) * cmax + 0x1p-15f * (rr + cmax * cmax) + 1e-30f;
      const float limit = best + band;
      // list this warp's candidates (row, codeword) of the stage: the scores
      // are read again (not held across the exchange) and turned into one
      // candidate mask per group before any list entry is written
      uint32_t cm[kMaxM / 16 / kColQ];
#pragma unroll
      for (int k = 0; k < kMaxM / 16 / kColQ; ++k) cm[k] = 0u;
#pragma unroll
      for (int k0 = 0; k0 < kMaxM / 16 / kColQ; k0 += 2) {
        if (cq + kColQ * k0 >= ngroups) break;
        uint32_t x[32];
        load_group_pair(base, cq, k0, ngroups, x);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int gi = cq + kColQ * (k0 + u);
          if (gi < ngroups) {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              cm[k0 + u] |= (cnorm[16 * gi + e] - 2.f * __uint_as_float(x[16 * u + e]) <= limit ? 1u : 0u) << e;
          }
        }
      }
#pragma unroll
      for (int k = 0; k < kMaxM / 16 / kColQ; ++k) {
        uint32_t cand = cm[k];
        while (cand) {
          const uint32_t m = (uint32_t)(16 * (cq + kColQ * k) + __ffs(cand) - 1);
          cand &= cand - 1;
          const uint32_t slot = atomicAdd(&ex->ncand, 1u);
          if (slot < (uint32_t)kCandCap) ex->cand[slot] = ((uint32_t)erow << 16) | m;
        }
      }
      tc::named_bar_sync(kBarAll, kRvqThreads);
      const uint32_t ncand = ex->ncand;
      int arg;
      if (ncand <= (uint32_t)kCandCap) {
        // every candidate's exact fp32 distance, four threads per candidate (a
        // quarter of the dimensions each); per row the smallest (distance,
        // codeword) key wins: lowest codeword on equal distances
        const int te = tid;
        for (uint32_t b0 = 0; b0 < 4 * ncand; b0 += (uint32_t)kRvqThreads) {
          const uint32_t i = b0 + (uint32_t)te;
          const bool live = i < 4 * ncand;
          const uint32_t pr = live ? ex->cand[i >> 2] : 0u;
          const int row = (int)(pr >> 16), m = (int)(pr & 0xFFFFu), qd = (int)(i & 3u);
          float dist = 0.f;
          if (live) {
            // the four lanes of a candidate (and the two candidates of a
            // quarter warp) start on different 16-byte chunks of their rows,
            // so their shared-memory reads fall on different banks
            const int rot = 2 * qd + ((te >> 2) & 1);
#pragma unroll
            for (int j = 0; j < kDq / 4; ++j) {
              const int c = qd * kDq + 4 * ((j + rot) % (kDq / 4));
              const float4 rv = *reinterpret_cast<const float4*>(R + sw_off(row, c, kRows));
              const float4 cv = *reinterpret_cast<const float4*>(C + sw_off(m, c, M));
              const float d0 = rv.x - cv.x, d1 = rv.y - cv.y, d2 = rv.z - cv.z, d3 = rv.w - cv.w;
              dist = fmaf(d0, d0, fmaf(d1, d1, fmaf(d2, d2, fmaf(d3, d3, dist))));
            }
          }
          // the four quarters of a candidate sit in four consecutive lanes;
          // summed in a fixed order (q0 + q1) + (q2 + q3)
          dist += __shfl_xor_sync(0xffffffffu, dist, 1);
          dist += __shfl_xor_sync(0xffffffffu, dist, 2);
          if (live && qd == 0)
            atomicMin(&ex->key[row], ((unsigned long long)__float_as_uint(dist) << 32) | (unsigned long long)m);
        }
        tc::named_bar_sync(kBarAll, kRvqThreads);
        const unsigned long long k = ex->key[erow];
        arg = k == ~0ull ? 0 : (int)(k & 0xFFFFFFFFull);
      } else {
        // more candidates than the list holds (near-equal codewords): each
        // warp re-scores its own groups' candidates row by row
        float exact_best = INFINITY;
        arg = INT_MAX;
        for (int gi = cq; gi < ngroups; gi += kColQ) {
          uint32_t x[32];
          KVC_TMEM_LD16(base + (uint32_t)(16 * gi), x);
          KVC_TMEM_WAIT_LD32(x);
          uint32_t cand = 0;
#pragma unroll
          for (int e = 0; e < 16; ++e) cand |= (cnorm[16 * gi + e] - 2.f * __uint_as_float(x[e]) <= limit ? 1u : 0u) << e;
          while (cand) {
            const int m = 16 * gi + __ffs(cand) - 1;  // ascending m
            cand &= cand - 1;
            float dist = 0.f;
#pragma unroll 8
            for (int c = 0; c < D; c += 4) {
              const float4 rv = *reinterpret_cast<const float4*>(R + sw_off(erow, c, kRows));
              const float4 cv = *reinterpret_cast<const float4*>(C + sw_off(m, c, M));
              const float d0 = rv.x - cv.x, d1 = rv.y - cv.y, d2 = rv.z - cv.z, d3 = rv.w - cv.w;
              dist = fmaf(d0, d0, fmaf(d1, d1, fmaf(d2, d2, fmaf(d3, d3, dist))));
            }
            if (dist < exact_best) {  // ascending m within this warp: ties keep the lowest index
              exact_best = dist;
              arg = m;
            }
          }
          __syncwarp();
        }
        ex->dist[cq][erow] = exact_best;
        ex->arg[cq][erow] = arg;
        tc::named_bar_sync(bar_id, 32 * kColQ);
        // the four parts' bests: smallest distance, lowest codeword on ties
        exact_best = ex->dist[0][erow];
        arg = ex->arg[0][erow];
#pragma unroll
        for (int q = 1; q < kColQ; ++q) {
          const float dq = ex->dist[q][erow];
          const int aq = ex->arg[q][erow];
          if (dq < exact_best || (dq == exact_best && aq < arg)) {
            exact_best = dq;
            arg = aq;
          }
        }
      }
      if (arg == INT_MAX) arg = 0;  // only a row whose scores are all NaN
      if (has_row && cq == 0) a.codes[(row0 + erow) * a.S + s] = arg;
      // residual update of this warp's quarter of the dimensions (rows past n
      // keep their zeros: code 0 is harmless)
      if (has_row) {
#pragma unroll
        for (int c = cq * kDq; c < (cq + 1) * kDq; c += 4) {
          float4* rp = reinterpret_cast<float4*>(R + sw_off(erow, c, kRows));
          const float4 cv = *reinterpret_cast<const float4*>(C + sw_off(arg, c, M));
          float4 rv = *rp;
          rv.x -= cv.x;
          rv.y -= cv.y;
          rv.z -= cv.z;
          rv.w -= cv.w;
          *rp = rv;
        }
      }
      tc::fence_proxy_async_smem();  // the new residual for the next stage's MMA
    }
    tc::tc_fence_before();
    __syncthreads();  // C and the scores are free
    tc::tc_fence_after();
  }

  if (bars->abort) {
    if (tid == 0) {
      // the copy and the MMAs of the stage that did not complete must land first
      if (cb_issued > stage_done) tc::mbar_drain(&bars->cb_full, (cb_issued - 1) & 1);
      if (mma_issued > stage_done) tc::mbar_drain(&bars->mma_done, (mma_issued - 1) & 1);
      set_dev_err(a.err, KVC_DEV_ERR_TIMEOUT);
    }
  } else if (a.residual != nullptr) {
    for (int i = tid; i < kRows * (D / 4); i += kRvqThreads) {
      const int row = i / (D / 4), c = (i % (D / 4)) * 4;
      if (row0 + row < a.n)
        *reinterpret_cast<float4*>(a.residual + (row0 + row) * D + c) =
            *reinterpret_cast<const float4*>(R + sw_off(row, c, kRows));
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kMaxM);
  }
}

kvc_status check_rvq(int64_t n, int32_t d, int32_t S, int32_t M) {
  if (d != 64 && d != 128) return fail(KVC_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  KVC_CHECK_ARG(n >= 0 && n < (int64_t(1) << 31), "n out of range");
  KVC_CHECK_ARG(S >= 1 && S <= kMaxS, "stages must be in 1..16");
  if (M < 16 || M > kMaxM || M % 16) return fail(KVC_ERR_UNSUPPORTED, "codebook size must be a multiple of 16 in 16..256");
  return KVC_OK;
}

}  // namespace
}  // namespace kvc

using namespace kvc;

extern "C" kvc_status kvc_rvq_encode(const uint16_t* x, int64_t x_stride, int64_t n, int32_t head_dim,
                                     const float* codebooks, int32_t stages, int32_t codebook_size, int32_t* codes,
                                     float* residual, int32_t* dev_err, void* stream) {
  clear_error();
  kvc_status s = check_rvq(n, head_dim, stages, codebook_size);
  if (s != KVC_OK) return s;
  KVC_CHECK_ARG(x && codebooks && codes, "x, codebooks and codes must be non-NULL");
  KVC_CHECK_ARG(x_stride >= head_dim, "x_stride must be >= head_dim");
  KVC_CHECK_ARG(aligned(codebooks, 16) && (!residual || aligned(residual, 16)),
                "codebooks and residual must be 16-byte aligned");
  if (n == 0) return KVC_OK;

  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  if (!encode) return fail(KVC_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  CUtensorMap cmap;
  cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)stages * codebook_size};
  cuuint64_t strides[1] = {(cuuint64_t)head_dim * 4};
  cuuint32_t box[2] = {32u, (cuuint32_t)codebook_size};
  cuuint32_t es[2] = {1u, 1u};
  if (encode(&cmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(codebooks), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return fail(KVC_ERR_CUDA, "cuTensorMapEncodeTiled failed for the codebooks");
  RvqArgs a{x, x_stride, n, stages, codebook_size, codes, residual, dev_err};
  static ContextCache cache;
  s = once_per_context(cache, [] {
    KVC_CUDA_TRY(cudaFuncSetAttribute(rvq_encode_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)RvqSmem<64>::kBytes));
    KVC_CUDA_TRY(cudaFuncSetAttribute(rvq_encode_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)RvqSmem<128>::kBytes));
    return KVC_OK;
  });
  if (s != KVC_OK) return s;
  const unsigned grid = (unsigned)((n + kRows - 1) / kRows);
  const size_t smem = head_dim == 128 ? RvqSmem<128>::kBytes : RvqSmem<64>::kBytes;
  const Launch l(dim3(grid), dim3(kRvqThreads), smem, (cudaStream_t)stream);
  if (head_dim == 128)
    KVC_CUDA_TRY(l.run(rvq_encode_kernel<128>, cmap, a));
  else
    KVC_CUDA_TRY(l.run(rvq_encode_kernel<64>, cmap, a));
  count_launch();
  return KVC_OK;
}
