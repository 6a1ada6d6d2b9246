// decode.cu -- attention of one decode query per head over the compacted cache.
//
// FastKV (gist.science 2502.01068) section 2.B: the K/V entries retained per
// KV head are the cache every later decoding step reads; section 1: decoding
// is bound by the bandwidth of reading that cache.  With the retained entries
// of KV head g in Kc[g], Vc[g] ([kk][d] each) and query head h of the group:
//     s_j = scale * q_h . Kc[g][j],   out_h = sum_j softmax(s)_j Vc[g][j].
//
// The G query heads of a KV head share every read of Kc[g] and Vc[g]; per
// retained entry the work is G*d multiply-adds for the logits and G*d for the
// output, a few FLOP per byte, so the kernel is an HBM stream on the CUDA
// cores (not a dense contraction: G = 4 query rows per KV head).  It is split
// over retained entries (flash-decoding): CTA (chunk, g) streams its chunk of
// Kc[g] / Vc[g] in 64-entry tiles through TMA (128-byte swizzle, so that one
// lane per entry reads its row without bank conflicts), keeps an online
// softmax per query head, and writes a partial (max, sum, output row); a
// second kernel, launched early (programmatic dependent launch) and waiting
// on the first, merges the partials of each head.
//
// A dedicated producer warp keeps the TMA ring full: it refills a stage as
// soon as the eight compute warps have released it, so loads of later tiles
// are in flight while the compute warps work on earlier ones (a refill
// issued by a compute warp would wait for the slowest warp of every tile).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include <cuda_bf16.h>

#include "common.cuh"
#include "tc.cuh"

namespace kvc {
namespace {

constexpr int kT = 64;             // retained entries per tile
constexpr int kDecThreads = 256;              // compute warps
constexpr int kDecBlock = kDecThreads + 32;   // + the producer warp
constexpr int kDecStages = 3;
constexpr int kDecMaxG = 16;       // query heads per KV head
constexpr int kDecCtaTarget = 296; // CTAs per launch: two per SM on 148 SMs
constexpr double kLog2e = 1.4426950408889634;

struct DecArgs {
  const uint16_t* q;  // [H][d] bf16, row stride q_sh
  int64_t q_sh;
  int64_t kk;         // retained entries per KV head
  int H, Hkv, G;
  int chunk;          // entries per CTA, a multiple of kT
  int nchunks;        // chunks per KV head
  float c;            // scale * log2(e)
  float* part_m;      // [H][nchunks]: running max (log2 domain)
  float* part_l;      // [H][nchunks]: sum of 2^(s*c - max)
  float* part_o;      // [H][nchunks][d]: sum of 2^(s*c - max) * v
  uint32_t* cnt;      // [Hkv]: chunks of the KV head done (tensor-core kernel; zero between calls)
  float* out;         // [H][d]
  int32_t* err;
};

template <int D>
struct DecSmem {
  static constexpr int kBoxes = D / 64;                      // 64-element (128-byte) column blocks
  static constexpr int kMatBytes = kBoxes * kT * 128;        // one K or V tile
  static constexpr int kStageBytes = 2 * kMatBytes;          // K tile, then V tile
  static constexpr size_t kFloats = (size_t)kDecMaxG * (D + 16) + (size_t)kDecMaxG * kT + 3 * kDecMaxG;
  static_assert((size_t)kDecStages * kStageBytes >= (size_t)(kDecThreads / 32) * kDecMaxG * (D + 2) * 4,
                "the merge of the warps reuses the stages");
  static constexpr size_t kBytes = 1024 + (size_t)kDecStages * kStageBytes + kFloats * 4 + 128;
};

// bf16 pair (low, high halves of w) -> two fp32 values
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// Byte offset of the 16-byte chunk k16 (0..7) of row j in a 128-byte
// swizzled TMA box of kT rows: chunks are XOR-ed with (row & 7).
__device__ __forceinline__ int sw128(int j, int k16) { return j * 128 + ((k16 ^ (j & 7)) << 4); }

// KG: query heads per KV head the kernel is built for (a.G <= KG; heads
// past a.G are zero padding whose outputs are dropped).
//
// Every warp owns 8 entries of each 64-entry tile from start to end: their
// logits (four lanes per entry, a quarter of the dimensions each), an online
// softmax per head over the warp's own entries, and the warp's output rows
// (four or two dimensions per lane).  No block-wide barrier runs per tile: a
// warp releases the stage through an mbarrier (one arrival per warp) and
// thread 0 refills it once all eight have.  The eight warps' (max, sum,
// output) are merged once at the end.
// Two CTAs per SM up to four heads per group; wider groups keep their
// per-head state in registers at one CTA per SM instead of spilling it.
template <int D, int KG>
__global__ void __launch_bounds__(kDecBlock, KG <= 4 ? 2 : 1)
decode_partial_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                      const DecArgs a) {
  using L = DecSmem<D>;
  constexpr int kWarps = kDecThreads / 32;       // 8
  constexpr int kPerWarp = kT / kWarps;          // entries per warp and tile (8)
  constexpr int kQuarter = D / 4;                // dimensions per logit lane
  constexpr int kQRow = D + 16;                  // floats per head of q (four padded quarters)
  constexpr int kQChunks = kQuarter / 8;         // 16-byte chunks per logit lane
  constexpr int kDL = D / 32;                    // output dimensions per lane (4 or 2)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stages = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* qs = reinterpret_cast<float*>(stages + (size_t)kDecStages * L::kStageBytes);  // [KG][D + 16]
  float* pw = qs + kDecMaxG * (D + 16);                    // [warp][kPerWarp][KG]: this tile's p
  uint64_t* full = reinterpret_cast<uint64_t*>(
      (reinterpret_cast<uintptr_t>(pw + kDecMaxG * kT) + 15) & ~uintptr_t(15));
  uint64_t* empty = full + kDecStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kDecStages);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.y, chunk = blockIdx.x;
  const int G = a.G;
  const int64_t e0 = (int64_t)chunk * a.chunk;
  const int64_t e1 = std::min<int64_t>(a.kk, e0 + a.chunk);
  const int ntiles = (int)((e1 - e0 + kT - 1) / kT);
  const int64_t row0 = (int64_t)g * a.kk + e0;  // first row of the chunk in the [Hkv*kk][D] view

  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], kWarps);
    }
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (tid == kDecThreads) {
    tc::prefetch_tmap(&kmap);
    tc::prefetch_tmap(&vmap);
  }
  __syncthreads();
  pdl_wait();  // Kc / Vc / q may come from the previous kernel of the stream
  // the merge kernel may launch now: it waits for this grid's completion
  pdl_trigger();

  auto issue = [&](int t) {
    const int s = t % kDecStages;
    uint8_t* dst = stages + (size_t)s * L::kStageBytes;
    tc::mbar_arrive_expect_tx(&full[s], (uint32_t)L::kStageBytes);
    const int y = (int)(row0 + (int64_t)t * kT);
#pragma unroll
    for (int cb = 0; cb < L::kBoxes; ++cb) {
      tc::tma_load_2d(dst + cb * kT * 128, &kmap, &full[s], cb * 64, y);
      tc::tma_load_2d(dst + L::kMatBytes + cb * kT * 128, &vmap, &full[s], cb * 64, y);
    }
  };
  const int je = lane >> 2, lq = lane & 3;  // logits: entry of the warp, quarter
  constexpr int kDP = kDL / 2;              // output dimension pairs per lane
  constexpr int kKG4 = (KG + 3) / 4;        // float4 groups of a p row
  float m_w[KG], l_w[KG];                   // this warp's running max and sum per head
  float2 o[KG][kDP];                        // this warp's output dims of this lane, per head
#pragma unroll
  for (int h = 0; h < KG; ++h) {
    m_w[h] = -INFINITY;
    l_w[h] = 0.f;
#pragma unroll
    for (int u = 0; u < kDP; ++u) o[h][u] = make_float2(0.f, 0.f);
  }
  float* pme = pw + warp * kPerWarp * (4 * kKG4);  // this warp's p block, rows padded to float4
  const int oe = kDL * lane, ocb = oe / 64, oe64 = oe % 64;

  int issued = 0;  // producer lane
  if (warp == kDecThreads / 32) {
    // ---- producer: the first stages at once, then each stage again as soon
    // as all compute warps have released it
    if (lane == 0) {
      for (; issued < ntiles; ++issued) {
        const int s = issued % kDecStages;
        if (issued >= kDecStages && !tc::mbar_wait(&empty[s], ((issued / kDecStages) - 1) & 1, abort_flag)) break;
        issue(issued);
      }
    }
  } else {
    // q as fp32, each head's D values in four quarters of D/4, every quarter
    // padded by 4 floats: the four lanes of an entry read their quarters at
    // different shared-memory banks (the stage loads are already in flight)
    for (int i = tid; i < KG * D; i += kDecThreads) {
      const int h = i / D, e = i % D;
      qs[h * kQRow + (e / kQuarter) * (kQuarter + 4) + e % kQuarter] =
          h < G ? __uint_as_float((uint32_t)a.q[(int64_t)(g * G + h) * a.q_sh + e] << 16) : 0.f;
    }
    tc::named_bar_sync(1, kDecThreads);
    for (int t = 0; t < ntiles; ++t) {
      const int s = t % kDecStages;
      if (!tc::mbar_wait(&full[s], (t / kDecStages) & 1, abort_flag)) break;
      const uint8_t* kt = stages + (size_t)s * L::kStageBytes;
      const uint8_t* vt = kt + L::kMatBytes;
      const int nvalid = (int)std::min<int64_t>(kT, e1 - (e0 + (int64_t)t * kT));
      const int jw = warp * kPerWarp;                       // the warp's first entry of the tile
      const int nw = max(0, min(kPerWarp, nvalid - jw));    // of which valid
      const int j = jw + je;

      // ---- logits of the warp's entries (log2 domain)
      float sc[KG];
      {
        float2 acc[KG];
#pragma unroll
        for (int h = 0; h < KG; ++h) acc[h] = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < kQChunks; ++c) {
          const int col = lq * kQuarter + c * 8;
          const uint4 kw = *reinterpret_cast<const uint4*>(kt + (col / 64) * kT * 128 + sw128(j, (col % 64) / 8));
          const float2 k0 = bf16x2_to_f2(kw.x), k1 = bf16x2_to_f2(kw.y), k2 = bf16x2_to_f2(kw.z),
                       k3 = bf16x2_to_f2(kw.w);
#pragma unroll
          for (int h = 0; h < KG; ++h) {
            const float* qh = qs + h * kQRow + lq * (kQuarter + 4) + c * 8;
            const float4 q0 = *reinterpret_cast<const float4*>(qh);
            const float4 q1 = *reinterpret_cast<const float4*>(qh + 4);
            float2 u = tc::fma2(k0, make_float2(q0.x, q0.y), acc[h]);
            u = tc::fma2(k1, make_float2(q0.z, q0.w), u);
            u = tc::fma2(k2, make_float2(q1.x, q1.y), u);
            acc[h] = tc::fma2(k3, make_float2(q1.z, q1.w), u);
          }
        }
#pragma unroll
        for (int h = 0; h < KG; ++h) {
          float v = acc[h].x + acc[h].y;
          v += __shfl_xor_sync(0xffffffffu, v, 1);
          v += __shfl_xor_sync(0xffffffffu, v, 2);
          sc[h] = je < nw ? v * a.c : -INFINITY;
        }
      }
      // ---- online softmax per head over the warp's entries
#pragma unroll
      for (int h = 0; h < KG; ++h) {
        float mx = sc[h];
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m_w[h], mx);
        const float al = m_w[h] == -INFINITY ? 0.f : tc::ex2_approx(m_w[h] - m_new);
        const float p = m_new == -INFINITY ? 0.f : tc::ex2_approx(sc[h] - m_new);
        float ps = p;
        ps += __shfl_xor_sync(0xffffffffu, ps, 4);
        ps += __shfl_xor_sync(0xffffffffu, ps, 8);
        ps += __shfl_xor_sync(0xffffffffu, ps, 16);
        l_w[h] = l_w[h] * al + ps;
        m_w[h] = m_new;
#pragma unroll
        for (int u = 0; u < kDP; ++u) o[h][u] = make_float2(o[h][u].x * al, o[h][u].y * al);
        if (lq == 0) pme[je * (4 * kKG4) + h] = p;
      }
      __syncwarp();
      // ---- the warp's output dims: o_h += sum over its entries of p_jh v_j
      const uint8_t* vrow = vt + ocb * kT * 128 + (oe64 & 7) * 2;
#pragma unroll 2
      for (int q = 0; q < nw; ++q) {
        const int jj = jw + q;
        float2 v[kDP];
        if constexpr (kDP == 2) {
          const uint2 w = *reinterpret_cast<const uint2*>(vrow + sw128(jj, oe64 >> 3));
          v[0] = bf16x2_to_f2(w.x);
          v[1] = bf16x2_to_f2(w.y);
        } else {
          v[0] = bf16x2_to_f2(*reinterpret_cast<const uint32_t*>(vrow + sw128(jj, oe64 >> 3)));
        }
        float pv[4 * kKG4];
#pragma unroll
        for (int b = 0; b < kKG4; ++b) {
          const float4 p4 = *reinterpret_cast<const float4*>(pme + q * (4 * kKG4) + 4 * b);
          pv[4 * b] = p4.x;
          pv[4 * b + 1] = p4.y;
          pv[4 * b + 2] = p4.z;
          pv[4 * b + 3] = p4.w;
        }
#pragma unroll
        for (int h = 0; h < KG; ++h)
#pragma unroll
          for (int u = 0; u < kDP; ++u) o[h][u] = tc::fma2(v[u], make_float2(pv[h], pv[h]), o[h][u]);
      }
      __syncwarp();  // every lane is done with the stage and p block
      if (lane == 0) tc::mbar_arrive(&empty[s]);
    }
  }  // compute warps
  __syncthreads();
  if (*abort_flag) {
    if (tid == kDecThreads) {
      // let the latest copy of every stage land before shared memory is released
      for (int u = max(0, issued - kDecStages); u < issued; ++u)
        tc::mbar_drain(&full[u % kDecStages], (u / kDecStages) & 1);
      set_dev_err(a.err, KVC_DEV_ERR_TIMEOUT);
    }
    return;
  }
  // ---- merge the eight compute warps (the stages are free now)
  float* wm = reinterpret_cast<float*>(stages);      // [warp][KG] max
  float* wl = wm + kWarps * KG;                      // [warp][KG] sum
  float* wo = wl + kWarps * KG;                      // [warp][KG][D] output rows
  if (warp < kWarps) {
    if (lane == 0)
#pragma unroll
      for (int h = 0; h < KG; ++h) {
        wm[warp * KG + h] = m_w[h];
        wl[warp * KG + h] = l_w[h];
      }
#pragma unroll
    for (int h = 0; h < KG; ++h)
#pragma unroll
      for (int u = 0; u < kDP; ++u) *reinterpret_cast<float2*>(wo + ((size_t)warp * KG + h) * D + oe + 2 * u) = o[h][u];
  }
  __syncthreads();
  for (int i = tid; i < G * D; i += kDecBlock) {
    const int h = i / D, e = i % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, wm[w * KG + h]);
    float O = 0.f, Lsum = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float mw = wm[w * KG + h];
      const float sc = mw == -INFINITY ? 0.f : tc::ex2_approx(mw - M);
      O += sc * wo[((size_t)w * KG + h) * D + e];
      Lsum += sc * wl[w * KG + h];
    }
    a.part_o[((size_t)(g * G + h) * a.nchunks + chunk) * D + e] = O;
    if (e == 0) {
      a.part_m[(size_t)(g * G + h) * a.nchunks + chunk] = M;
      a.part_l[(size_t)(g * G + h) * a.nchunks + chunk] = Lsum;
    }
  }
}

// --------------------------------------------------------------------------
// tcgen05 variant (head_dim 128, up to 8 query heads per KV head).  The two
// contractions of a 128-entry tile run on the tensor cores, so the CUDA cores
// only form the probabilities and the stream of Kc / Vc sets the pace:
//   logits  S[entry][h] = Kc_tile (M = 128 entries, K = d) x q^T (N = 16: the
//           group's heads, zero rows past G), fp32 in TMEM;
//   output  O[dim][n]   = Vc_tile^T (M = d = 128, K = entries; the TMA tile of
//           Vc read as an MN-major operand) x P (N = 16, K = entries), where
//           P rows 0..7 hold bf16(p_h) and rows 8..15 the bf16 rounding
//           residual p_h - bf16(p_h), so hi + lo carries p_h to ~2^-17.
// Each epilogue warp owns 32 entries of a tile and a running reference per
// head (the max logit its entries have shown, log2 domain), so no barrier
// joins the warps inside the loop; the output MMA of a tile is split into the
// four warps' 32-entry slices, each into its own TMEM accumulator, and every
// epilogue thread (one output dimension) folds the four slices into its
// registers with the four references.
// Kc and Vc tiles stream through two rings: a Kc tile is released as soon as
// its logits MMA has read it, a Vc tile only after the output MMA, which
// waits for the probabilities.
// Warp roles: 0 Kc producer, 1 TMEM allocator + MMA issuer, 2..5 epilogue
// (TMEM lane quarter = warp & 3), 6 Vc producer.
// --------------------------------------------------------------------------
constexpr int kTcT = 128;        // entries per tile (MMA M of the logits)
constexpr int kTcKStages = 1;    // 32 KB Kc tiles (held only until the logits MMA)
constexpr int kTcVStages = 2;    // 32 KB Vc tiles (held until the output MMA)
constexpr int kTcCtasPerSm = 2;  // 110 KB of shared memory and 256 TMEM columns each
constexpr float kTcSlack = 8.f;  // log2 units a logit may pass a warp's reference by
constexpr int kTcMaxG = 8;
constexpr int kTcBlock = 224;
constexpr uint32_t kTcCols = 256;  // S: 2 x 16 columns, O: 2 buffers x 4 slices x 16
constexpr uint32_t kTcO = 32;      // first O column

struct TcSmem {
  static constexpr int kTile = kTcT * 128;           // one 64-column block of a tile (16 KB)
  static constexpr int kStage = 2 * kTile;           // a Kc or a Vc tile (two column blocks)
  static constexpr int kQ = 2 * 16 * 128;            // q: 2 column blocks x 16 rows x 128 B
  static constexpr int kP = 2 * 16 * 128;            // one P buffer: 2 entry blocks x 16 rows x 128 B
  static constexpr int kVOff = kTcKStages * kStage;  // the Vc ring follows the Kc ring
  static constexpr int kQOff = kVOff + kTcVStages * kStage;
  static constexpr int kPOff = kQOff + kQ;
  static constexpr int kBarOff = kPOff + 2 * kP;
  static constexpr size_t kBytes = 1024 + (size_t)kBarOff + 1024;
};

struct TcBars {
  uint64_t kfull[kTcKStages], kempty[kTcKStages], vfull[kTcVStages], vempty[kTcVStages];
  uint64_t s_full[2], s_empty[2], p_full[2], o_full[2], o_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  int last;  // this CTA took the KV head's last ticket: it merges the partials
  // reference each warp used for the P rows of tile t, at [t & 3]: a warp can
  // run at most two tiles ahead of the slowest one (the logits buffer of tile
  // t + 2 is released only once every warp has read tile t's), so a slot is
  // rewritten only after every warp has folded the tile it belonged to
  float mref[4][4][kTcMaxG];
  float wm[4][kTcMaxG], wl[4][kTcMaxG];
};

// Byte offset of bf16 element (row r, column k) in a K-major operand stored
// as 64-column blocks of `rows` rows x 128 B with the 128-byte swizzle.
__device__ __forceinline__ int kmaj_off(int r, int k, int rows) {
  return (k >> 6) * rows * 128 + r * 128 + ((((k & 63) >> 3) ^ (r & 7)) << 4) + ((k & 7) << 1);
}

// MN-major operand descriptor, 128-byte swizzle: 64 MN-consecutive elements per
// 128-byte row, K rows at 128 B; `lbo` bytes between 64-element MN blocks,
// 1024 B between 8-row K groups.
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t smem_addr, uint32_t lbo) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

template <int KG>
__global__ void __launch_bounds__(kTcBlock, kTcCtasPerSm)
decode_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                 const DecArgs a) {
  using L = TcSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qb = sm + L::kQOff;
  uint8_t* pb = sm + L::kPOff;
  TcBars* bars = reinterpret_cast<TcBars*>(sm + L::kBarOff);
  static_assert(sizeof(TcBars) <= 1024, "barrier block");

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.y, chunk = blockIdx.x;
  const int G = a.G;
  const int64_t e0 = (int64_t)chunk * a.chunk;
  const int64_t e1 = std::min<int64_t>(a.kk, e0 + a.chunk);
  const int ntiles = (int)((e1 - e0 + kTcT - 1) / kTcT);
  const int64_t row0 = (int64_t)g * a.kk + e0;

  if (tid == 0) {
    for (int s = 0; s < kTcKStages; ++s) {
      tc::mbar_init(&bars->kfull[s], 1);
      tc::mbar_init(&bars->kempty[s], 1);
    }
    for (int s = 0; s < kTcVStages; ++s) {
      tc::mbar_init(&bars->vfull[s], 1);
      tc::mbar_init(&bars->vempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&bars->s_full[b], 1);
      tc::mbar_init(&bars->s_empty[b], 4);
      tc::mbar_init(&bars->p_full[b], 4);
      tc::mbar_init(&bars->o_full[b], 1);
      tc::mbar_init(&bars->o_empty[b], 4);
    }
    tc::mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) tc::prefetch_tmap(&kmap);
  if (warp == 6 && lane == 0) tc::prefetch_tmap(&vmap);
  if (warp == 1) {
    tc::tmem_alloc(&bars->tmem_base, kTcCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  pdl_wait();  // Kc / Vc / q may come from the previous kernel of the stream
  pdl_trigger();
  if (warp >= 1 && warp <= 5) {
    // while the producers start the streams: both P buffers zero (rows past
    // the group stay zero), and q of the group as the logits' B operand
    // (rows = heads, zero past G; K = d)
    constexpr int kN = 160;
    for (int i = tid - 32; i < 2 * L::kP / 16; i += kN) reinterpret_cast<uint4*>(pb)[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int i = tid - 32; i < 16 * 128; i += kN) {
      const int h = i >> 7, k = i & 127;
      const uint16_t v = h < G ? a.q[(int64_t)(g * G + h) * a.q_sh + k] : (uint16_t)0;
      *reinterpret_cast<uint16_t*>(qb + kmaj_off(h, k, 16)) = v;
    }
    tc::fence_proxy_async_smem();
    tc::named_bar_sync(1, kN);
  }
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;
  float o_r[KG];  // epilogue: this thread's output dimension per head (relative to m_acc)
#pragma unroll
  for (int h = 0; h < KG; ++h) o_r[h] = 0.f;

  if (warp == 0 || warp == 6) {
    // ---- TMA producers: warp 0 the Kc tiles, warp 6 the Vc tiles
    if (lane == 0) {
      const bool is_k = warp == 0;
      const int ns = is_k ? kTcKStages : kTcVStages;
      uint64_t* fullb = is_k ? bars->kfull : bars->vfull;
      uint64_t* emptyb = is_k ? bars->kempty : bars->vempty;
      uint8_t* ring = sm + (is_k ? 0 : L::kVOff);
      const CUtensorMap* map = is_k ? &kmap : &vmap;
      int issued = 0;
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % ns;
        if (t >= ns && !tc::mbar_wait(&emptyb[s], ((t / ns) - 1) & 1, abort_flag)) break;
        tc::mbar_arrive_expect_tx(&fullb[s], (uint32_t)L::kStage);
        uint8_t* dst = ring + (size_t)s * L::kStage;
        const int y = (int)(row0 + (int64_t)t * kTcT);
        tc::tma_load_2d(dst, map, &fullb[s], 0, y);
        tc::tma_load_2d(dst + L::kTile, map, &fullb[s], 64, y);
        issued = t + 1;
      }
      if (*abort_flag)
        for (int t = std::max(0, issued - ns); t < issued; ++t) tc::mbar_drain(&fullb[t % ns], (t / ns) & 1);
    }
  } else if (warp == 1) {
    // ---- MMA issuer: logits of tile t, then the output of tile t - 1
    if (lane == 0) {
      const uint32_t id_s = tc::idesc_bf16_f32(128, 16);
      const uint32_t id_o = tc::idesc_bf16_f32(128, 16) | (1u << 15);  // A (Vc^T) MN-major
      const uint64_t q_desc = tc::desc_k_sw128(tc::smem_u32(qb));
      const uint64_t k_desc = tc::desc_k_sw128(tc::smem_u32(sm));
      const uint64_t v_desc = desc_mn_sw128(tc::smem_u32(sm + L::kVOff), (uint32_t)L::kTile);
      const uint64_t p_desc = tc::desc_k_sw128(tc::smem_u32(pb));
      auto logits = [&](int t) -> bool {
        const int s = t % kTcKStages, b = t & 1;
        if (!tc::mbar_wait(&bars->kfull[s], (t / kTcKStages) & 1, abort_flag)) return false;
        if (t >= 2 && !tc::mbar_wait(&bars->s_empty[b], ((t >> 1) - 1) & 1, abort_flag)) return false;
        tc::tc_fence_after();
        const uint64_t kd = k_desc + (uint64_t)(((uint32_t)s * L::kStage) >> 4);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = (uint32_t)((ks >> 2) * L::kTile + (ks & 3) * 32) >> 4;  // K tile: 64-col block, 32 B step
          const uint32_t qoff = (uint32_t)((ks >> 2) * 2048 + (ks & 3) * 32) >> 4;    // q: 16-row blocks of 2 KB
          tc::mma_bf16(tmem + (uint32_t)(16 * b), kd + off, q_desc + qoff, id_s, ks != 0);
        }
        tc::mma_commit(&bars->s_full[b]);
        tc::mma_commit(&bars->kempty[s]);  // the Kc tile is read
        return true;
      };
      auto output = [&](int t) -> bool {
        const int s = t % kTcVStages, b = t & 1;
        if (!tc::mbar_wait(&bars->vfull[s], (t / kTcVStages) & 1, abort_flag)) return false;
        if (!tc::mbar_wait(&bars->p_full[b], (t >> 1) & 1, abort_flag)) return false;
        if (t >= 2 && !tc::mbar_wait(&bars->o_empty[b], ((t >> 1) - 1) & 1, abort_flag)) return false;
        tc::tc_fence_after();
        const uint64_t vd = v_desc + (uint64_t)(((uint32_t)s * L::kStage) >> 4);
        const uint64_t pd = p_desc + (uint64_t)(((uint32_t)b * L::kP) >> 4);
#pragma unroll
        for (int w = 0; w < 4; ++w)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int en = 32 * w + 16 * j;  // first entry of this K step
            const uint32_t voff = (uint32_t)(en * 128) >> 4;                          // 16 Vc rows = 2 KB
            const uint32_t poff = (uint32_t)((en >> 6) * 2048 + (en & 63) * 2) >> 4;  // P: 64-entry blocks
            tc::mma_bf16(tmem + kTcO + (uint32_t)(64 * b + 16 * w), vd + voff, pd + poff, id_o, j != 0);
          }
        tc::mma_commit(&bars->o_full[b]);
        tc::mma_commit(&bars->vempty[s]);  // the Vc tile is read
        return true;
      };
      bool ok = true;
      for (int t = 0; ok && t <= ntiles; ++t) {
        if (t < ntiles) ok = logits(t);
        if (ok && t >= 1) ok = output(t - 1);
      }
      tc::mma_commit(&bars->mma_done);  // every MMA issued above has completed before TMEM is freed
      tc::mbar_drain(&bars->mma_done, 0);
    }
  } else {
    // ---- epilogue: warp quarter wq owns entries 32 wq .. 32 wq + 31 of each
    // tile (softmax role) and output dimension 32 wq + lane (output role)
    const int wq = warp & 3;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * wq) << 16);
    float m_w[KG], l_t[KG], m_acc[KG];
#pragma unroll
    for (int h = 0; h < KG; ++h) {
      m_w[h] = -INFINITY;
      l_t[h] = 0.f;
      m_acc[h] = -INFINITY;
    }
    bool ok = true;
    for (int t = 0; ok && t <= ntiles; ++t) {
      if (t < ntiles) {
        const int b = t & 1;
        if (!tc::mbar_wait(&bars->s_full[b], (t >> 1) & 1, abort_flag)) { ok = false; break; }
        tc::tc_fence_after();
        uint32_t x[32];
        KVC_TMEM_LD16(lane_base + (uint32_t)(16 * b), x);
        KVC_TMEM_WAIT_LD32(x);
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bars->s_empty[b]);
        const int ent = 32 * wq + lane;
        const bool valid = (int64_t)t * kTcT + ent < e1 - e0;
        uint8_t* pbb = pb + b * L::kP;
#pragma unroll
        for (int h = 0; h < KG; ++h) {
          const float sv = valid && h < G ? __uint_as_float(x[h]) * a.c : -INFINITY;
          // the reference moves (to the warp's max) only when a logit passes it
          // by more than kTcSlack: p <= 2^kTcSlack otherwise, which bf16 and the
          // fp32 sums carry exactly as well as p <= 1 (warp-uniform vote)
          if (__any_sync(0xffffffffu, sv > m_w[h] + kTcSlack)) {
            float mx = sv;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            l_t[h] *= m_w[h] == -INFINITY ? 0.f : tc::ex2_approx(m_w[h] - mx);
            m_w[h] = mx;
          }
          const float p = m_w[h] == -INFINITY ? 0.f : tc::ex2_approx(sv - m_w[h]);
          l_t[h] += p;
          const __nv_bfloat16 hi = __float2bfloat16_rn(p);
          const __nv_bfloat16 lo = __float2bfloat16_rn(p - __bfloat162float(hi));
          if (h < G) {
            *reinterpret_cast<__nv_bfloat16*>(pbb + kmaj_off(h, ent, 16)) = hi;
            *reinterpret_cast<__nv_bfloat16*>(pbb + kmaj_off(8 + h, ent, 16)) = lo;
          }
          if (lane == 0) bars->mref[t & 3][wq][h] = m_w[h];
        }
        tc::fence_proxy_async_smem();  // P visible to the tensor core
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bars->p_full[b]);
      }
      if (t >= 1) {
        // fold the output slices of tile t - 1 into this thread's dimension
        const int tp = t - 1, b = tp & 1;
        // the slices' references: written by each warp before its P arrival
        if (!tc::mbar_wait(&bars->p_full[b], (tp >> 1) & 1, abort_flag)) { ok = false; break; }
        if (!tc::mbar_wait(&bars->o_full[b], (tp >> 1) & 1, abort_flag)) { ok = false; break; }
        tc::tc_fence_after();
        uint32_t y[64];
        KVC_TMEM_LD64(lane_base + kTcO + (uint32_t)(64 * b), y);
        KVC_TMEM_WAIT_LD64(y);
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bars->o_empty[b]);
#pragma unroll
        for (int h = 0; h < KG; ++h) {
          if (h >= G) continue;
          float mr[4], mt = m_acc[h];
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            mr[w] = bars->mref[tp & 3][w][h];
            mt = fmaxf(mt, mr[w]);
          }
          if (mt == -INFINITY) continue;
          float acc = m_acc[h] == -INFINITY ? 0.f : o_r[h] * tc::ex2_approx(m_acc[h] - mt);
#pragma unroll
          for (int w = 0; w < 4; ++w)
            if (mr[w] != -INFINITY)
              acc += (__uint_as_float(y[16 * w + h]) + __uint_as_float(y[16 * w + 8 + h])) * tc::ex2_approx(mr[w] - mt);
          o_r[h] = acc;
          m_acc[h] = mt;
        }
      }
    }
    if (ok) {
      // this warp's (reference, sum) per head for the CTA merge
#pragma unroll
      for (int h = 0; h < KG; ++h) {
        float l = l_t[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (lane == 0) {
          bars->wm[wq][h] = m_w[h];
          bars->wl[wq][h] = l;
        }
      }
    }
  }
  __syncthreads();
  if (*abort_flag) {
    if (tid == 0) set_dev_err(a.err, KVC_DEV_ERR_TIMEOUT);
  } else if (warp >= 2 && warp <= 5) {
    const int wq = warp & 3;
    const int dim = 32 * wq + lane;
#pragma unroll
    for (int h = 0; h < KG; ++h) {
      if (h >= G) break;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w) M = fmaxf(M, bars->wm[w][h]);
      float Lsum = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w)
        if (bars->wm[w][h] != -INFINITY) Lsum += bars->wl[w][h] * tc::ex2_approx(bars->wm[w][h] - M);
      const size_t slot = (size_t)(g * G + h) * a.nchunks + chunk;
      a.part_o[slot * 128 + dim] = o_r[h];
      if (dim == 0) {
        a.part_m[slot] = M;
        a.part_l[slot] = Lsum;
      }
    }
  }
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTcCols);
  }
  // ---- the last CTA of the KV head to finish merges the chunk partials of
  // its G heads (out_h = sum_c 2^(m_c - M) o_c / sum_c 2^(m_c - M) l_c).  A CTA
  // that gave up on a wait still takes its ticket, so the counter always
  // returns to zero (the output is then flagged by the timeout bit).
  __threadfence();
  __syncthreads();
  if (tid == 0) bars->last = atomicAdd(&a.cnt[g], 1u) == (uint32_t)(a.nchunks - 1);
  __syncthreads();
  if (!bars->last) return;
  __threadfence();
  // One warp per head of the group, lane l = output dimensions 4l .. 4l + 3.
  // The rows of the first 16 chunks are requested together with the chunk
  // references and sums (one round trip to L2), the weights 2^(m_c - M) and
  // the normaliser are formed from those, and the remaining rows follow in
  // batches of 16.  Chunk references and sums are staged in the stage memory,
  // which no copy or MMA uses any more.  Sums run over the chunks in order.
  const int nch = a.nchunks;
  float* wv = reinterpret_cast<float*>(sm);  // [G][nch]: references, then weights
  float* lsm = wv + G * nch;                 // [G][nch]: sums
  for (int hl = warp; hl < G; hl += kTcBlock / 32) {
    const float* pm = a.part_m + (size_t)(g * G + hl) * nch;
    const float* pl = a.part_l + (size_t)(g * G + hl) * nch;
    const float4* po = reinterpret_cast<const float4*>(a.part_o + (size_t)(g * G + hl) * nch * 128) + lane;
    float* wh = wv + hl * nch;
    float* lh = lsm + hl * nch;
    float4 v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) v[u] = u < nch ? __ldcg(po + (size_t)u * 32) : make_float4(0.f, 0.f, 0.f, 0.f);
    float M = -INFINITY;
    for (int c = lane; c < nch; c += 32) {
      const float mc = __ldcg(pm + c);
      wh[c] = mc;
      lh[c] = __ldcg(pl + c);
      M = fmaxf(M, mc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float Ls = 0.f;
    for (int c = lane; c < nch; c += 32) {
      const float mc = wh[c];
      const float wc = mc == -INFINITY ? 0.f : tc::ex2_approx(mc - M);
      wh[c] = wc;
      Ls += wc * lh[c];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
    __syncwarp();  // every lane's weights are in shared memory
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c0 = 0; c0 < nch; c0 += 16) {
      if (c0 > 0) {
#pragma unroll
        for (int u = 0; u < 16; ++u)
          v[u] = c0 + u < nch ? __ldcg(po + (size_t)(c0 + u) * 32) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const float wc = c0 + u < nch ? wh[c0 + u] : 0.f;
        acc.x += wc * v[u].x;
        acc.y += wc * v[u].y;
        acc.z += wc * v[u].z;
        acc.w += wc * v[u].w;
      }
    }
    *reinterpret_cast<float4*>(a.out + (size_t)(g * G + hl) * 128 + 4 * lane) =
        make_float4(acc.x / Ls, acc.y / Ls, acc.z / Ls, acc.w / Ls);
  }
  if (tid == 0) a.cnt[g] = 0u;
}

// Merge the chunk partials of head h: out = sum_c 2^(m_c - M) o_c / sum_c 2^(m_c - M) l_c.
// The chunk weights are formed once (shared memory), then every thread sums
// its dimension over the chunks with the loads of eight chunks in flight.
constexpr int kMaxChunks = 1024;
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const DecArgs a) {
  __shared__ float wsh[kMaxChunks];
  __shared__ float red[D / 32];
  __shared__ float msh;
  pdl_wait();
  const int h = blockIdx.x, e = threadIdx.x, lane = e & 31, warp = e >> 5;
  const int nch = a.nchunks;
  const float* pm = a.part_m + (size_t)h * nch;
  const float* pl = a.part_l + (size_t)h * nch;
  float mx = -INFINITY;
  for (int c = e; c < nch; c += D) mx = fmaxf(mx, pm[c]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  if (e == 0) {
    float m = red[0];
    for (int w = 1; w < D / 32; ++w) m = fmaxf(m, red[w]);
    msh = m;
  }
  __syncthreads();
  const float M = msh;
  float lsum = 0.f;
  for (int c = e; c < nch; c += D) {
    const float w = pm[c] == -INFINITY ? 0.f : tc::ex2_approx(pm[c] - M);
    wsh[c] = w;
    lsum += w * pl[c];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
  __syncthreads();  // wsh complete; red reused below
  if (lane == 0) red[warp] = lsum;
  __syncthreads();
  float L = 0.f;
  for (int w = 0; w < D / 32; ++w) L += red[w];
  const float* po = a.part_o + (size_t)h * nch * D + e;
  float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  int c = 0;
  for (; c + 8 <= nch; c += 8) {
#pragma unroll
    for (int u = 0; u < 8; ++u) o[u] += wsh[c + u] * po[(size_t)(c + u) * D];
  }
  for (; c < nch; ++c) o[0] += wsh[c] * po[(size_t)c * D];
  a.out[(size_t)h * D + e] = (((o[0] + o[1]) + (o[2] + o[3])) + ((o[4] + o[5]) + (o[6] + o[7]))) / L;
}

// The tensor-core kernel serves head_dim 128 with up to 8 query heads per KV
// head; the CUDA-core kernel everything else.
bool decode_on_tc(int G, int d) { return d == 128 && G <= kTcMaxG; }

// Entries per tile of the kernel that serves (G, d).
int decode_tile(int G, int d) { return decode_on_tc(G, d) ? kTcT : kT; }

// Chunks per KV head: about one wave of CTAs (one per SM for the tensor-core
// kernel, two for the CUDA-core one), never more than one per tile.
int decode_chunks(int64_t kk, int Hkv, int G, int d) {
  const int tile = decode_tile(G, d);
  const int target = decode_on_tc(G, d) ? kTcCtasPerSm * num_sms() : kDecCtaTarget;
  const int64_t tiles = (kk + tile - 1) / tile;
  const int64_t want = std::min<int64_t>(kMaxChunks, std::max<int64_t>(1, target / Hkv));
  const int64_t per = (tiles + std::min(tiles, want) - 1) / std::min(tiles, want);  // tiles per chunk
  return (int)((tiles + per - 1) / per);
}

// Query heads per KV head the kernel is instantiated for: the group size, or
// the next instantiated size above it (the extra heads are zero padding).
int decode_group_slots(int G) {
  if (G <= 6) return G;
  return G <= 8 ? 8 : 16;
}

template <int D, int KG>
kvc_status launch_decode_g(const Launch& l, const CUtensorMap (&maps)[2], const DecArgs& a) {
  static ContextCache cache;
  kvc_status s = once_per_context(cache, [] {
    KVC_CUDA_TRY(cudaFuncSetAttribute(decode_partial_kernel<D, KG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)DecSmem<D>::kBytes));
    return KVC_OK;
  });
  if (s != KVC_OK) return s;
  KVC_CUDA_TRY(l.run(decode_partial_kernel<D, KG>, maps[0], maps[1], a));
  return KVC_OK;
}

template <int KG>
kvc_status launch_decode_tc(const Launch& l, const CUtensorMap (&maps)[2], const DecArgs& a) {
  static ContextCache cache;
  kvc_status s = once_per_context(cache, [] {
    KVC_CUDA_TRY(cudaFuncSetAttribute(decode_tc_kernel<KG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)TcSmem::kBytes));
    return KVC_OK;
  });
  if (s != KVC_OK) return s;
  KVC_CUDA_TRY(l.run(decode_tc_kernel<KG>, maps[0], maps[1], a));
  return KVC_OK;
}

template <int D>
kvc_status launch_decode(const Launch& l, int kg, const CUtensorMap (&maps)[2], const DecArgs& a) {
  switch (kg) {
    case 1: return launch_decode_g<D, 1>(l, maps, a);
    case 2: return launch_decode_g<D, 2>(l, maps, a);
    case 3: return launch_decode_g<D, 3>(l, maps, a);
    case 4: return launch_decode_g<D, 4>(l, maps, a);
    case 5: return launch_decode_g<D, 5>(l, maps, a);
    case 6: return launch_decode_g<D, 6>(l, maps, a);
    case 8: return launch_decode_g<D, 8>(l, maps, a);
    default: return launch_decode_g<D, 16>(l, maps, a);
  }
}

kvc_status check_decode(int32_t H, int32_t Hkv, int32_t d, int64_t kk) {
  KVC_CHECK_ARG(H >= 1 && Hkv >= 1 && H % Hkv == 0, "num_heads must be a positive multiple of num_kv_heads");
  if (d != 64 && d != 128) return fail(KVC_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (H / Hkv > kDecMaxG) return fail(KVC_ERR_UNSUPPORTED, "at most 16 query heads per KV head");
  KVC_CHECK_ARG(kk >= 1 && kk * (int64_t)Hkv < (int64_t(1) << 31), "need 1 <= kk and kk * num_kv_heads < 2^31");
  return KVC_OK;
}

size_t decode_ws_bytes(int32_t H, int32_t Hkv, int32_t d, int64_t kk) {
  const size_t nch = (size_t)decode_chunks(kk, Hkv, H / Hkv, d);
  return round_up((size_t)Hkv * 4, kWsAlign) + round_up((size_t)H * nch * 4, kWsAlign) * 2 +
         round_up((size_t)H * nch * d * 4, kWsAlign);
}

}  // namespace
}  // namespace kvc

using namespace kvc;

extern "C" kvc_status kvc_decode_workspace_size(int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                                                int64_t kk, size_t* bytes) {
  clear_error();
  kvc_status s = check_decode(num_heads, num_kv_heads, head_dim, kk);
  if (s != KVC_OK) return s;
  KVC_CHECK_ARG(bytes != nullptr, "bytes must be non-NULL");
  *bytes = decode_ws_bytes(num_heads, num_kv_heads, head_dim, kk);
  return KVC_OK;
}

extern "C" kvc_status kvc_decode_attention(const uint16_t* q, int64_t q_stride_h, const uint16_t* k_c,
                                           const uint16_t* v_c, int64_t kk, int32_t num_heads,
                                           int32_t num_kv_heads, int32_t head_dim, float scale, float* out,
                                           void* ws, size_t ws_bytes, int32_t* dev_err, void* stream) {
  clear_error();
  kvc_status s = check_decode(num_heads, num_kv_heads, head_dim, kk);
  if (s != KVC_OK) return s;
  KVC_CHECK_ARG(q && k_c && v_c && out, "q, k_c, v_c and out must be non-NULL");
  KVC_CHECK_ARG(aligned(k_c, 16) && aligned(v_c, 16) && aligned(out, 16), "k_c, v_c and out must be 16-byte aligned");
  KVC_CHECK_ARG(q_stride_h >= head_dim, "q_stride_h must be >= head_dim");
  KVC_CHECK_ARG(scale > 0.f && scale < 1e30f, "scale must be positive and finite");
  const size_t need = decode_ws_bytes(num_heads, num_kv_heads, head_dim, kk);
  if (!ws || ws_bytes < need || !aligned(ws, kWsAlign))
    return fail(KVC_ERR_WORKSPACE, "decode workspace missing, too small or not 256-B aligned");

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
  const int d = head_dim, Hkv = num_kv_heads, G = num_heads / num_kv_heads;
  const bool on_tc = decode_on_tc(G, d);
  const int tile = decode_tile(G, d);
  CUtensorMap maps[2];
  const uint16_t* srcs[2] = {k_c, v_c};
  for (int i = 0; i < 2; ++i) {
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)(kk * Hkv)};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {64u, (cuuint32_t)tile};
    cuuint32_t es[2] = {1u, 1u};
    if (encode(&maps[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(srcs[i]), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return fail(KVC_ERR_CUDA, "cuTensorMapEncodeTiled failed for the compacted cache");
  }
  DecArgs a{};
  a.q = q;
  a.q_sh = q_stride_h;
  a.kk = kk;
  a.H = num_heads;
  a.Hkv = Hkv;
  a.G = num_heads / Hkv;
  a.nchunks = decode_chunks(kk, Hkv, G, d);
  const int64_t tiles = (kk + tile - 1) / tile;
  a.chunk = (int)(((tiles + a.nchunks - 1) / a.nchunks) * tile);
  a.c = (float)((double)scale * kLog2e);
  WsCursor wc{static_cast<char*>(ws), ws_bytes};
  a.cnt = wc.take<uint32_t>((size_t)Hkv);
  a.part_m = wc.take<float>((size_t)num_heads * a.nchunks);
  a.part_l = wc.take<float>((size_t)num_heads * a.nchunks);
  a.part_o = wc.take<float>((size_t)num_heads * a.nchunks * d);
  if (!wc.ok) return fail(KVC_ERR_WORKSPACE, "decode workspace too small");
  a.out = out;
  a.err = dev_err;

  const int kg = decode_group_slots(a.G);
  const cudaStream_t st = (cudaStream_t)stream;
  if (on_tc) {  // one launch: the last CTA of each KV head merges
    const Launch l(dim3((unsigned)a.nchunks, (unsigned)Hkv), dim3(kTcBlock), TcSmem::kBytes, st);
    s = G <= 4 ? launch_decode_tc<4>(l, maps, a) : launch_decode_tc<8>(l, maps, a);
    if (s != KVC_OK) return s;
    count_launch(1);
    return KVC_OK;
  } else {
    const size_t smem = d == 128 ? DecSmem<128>::kBytes : DecSmem<64>::kBytes;
    const Launch l(dim3((unsigned)a.nchunks, (unsigned)Hkv), dim3(kDecBlock), smem, st);
    s = d == 128 ? launch_decode<128>(l, kg, maps, a) : launch_decode<64>(l, kg, maps, a);
    if (s != KVC_OK) return s;
  }
  {
    const Launch l(dim3((unsigned)num_heads), dim3((unsigned)d), 0, st);
    if (d == 128)
      KVC_CUDA_TRY(l.run(decode_combine_kernel<128>, a));
    else
      KVC_CUDA_TRY(l.run(decode_combine_kernel<64>, a));
  }
  count_launch(2);
  return KVC_OK;
}
