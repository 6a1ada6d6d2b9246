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
// Warp 0 issues TMA and MMA (lane 0); warps 1..4 own one row per thread (TMEM
// lane = row).  Every wait is bounded; on a timeout the CTA records
// KVC_DEV_ERR_TIMEOUT, lets its copies and MMAs land, frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "tc.cuh"

namespace kvc {
namespace {

constexpr int kRows = 128;       // rows per CTA (MMA M)
constexpr int kRvqThreads = 160; // warp 0: TMA + MMA; warps 1..4: one row per thread
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
  static constexpr size_t kBytes = 1024 + kRBytes + kCBytes + kMaxM * 4 + 256;
};

// Byte offset of the 16-byte chunk holding elements c..c+3 (c % 4 == 0) of
// row `row` in a K-major SW128 matrix of `rows` rows.
__device__ __forceinline__ uint32_t sw_off(int row, int c, int rows) {
  const int blk = c >> 5, k16 = (c & 31) >> 2;
  return (uint32_t)(blk * rows * 128 + row * 128 + ((k16 ^ (row & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(kRvqThreads, 1)
rvq_encode_kernel(const __grid_constant__ CUtensorMap cmap, const RvqArgs a) {
  using L = RvqSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* R = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* C = R + L::kRBytes;
  float* cnorm = reinterpret_cast<float*>(C + L::kCBytes);
  RvqBars* bars = reinterpret_cast<RvqBars*>(cnorm + kMaxM);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t row0 = (int64_t)blockIdx.x * kRows;
  const int M = a.M;
  if (tid == 0) {
    tc::mbar_init(&bars->cb_full, 1);
    tc::mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    tc::fence_mbar_init();
    tc::prefetch_tmap(&cmap);
  }
  if (warp == 0) {
    tc::tmem_alloc(&bars->tmem_base, kMaxM);
    tc::tmem_relinquish();
  }
  pdl_wait();  // the rows may come from the previous kernel of the stream
  // rows -> fp32 residual (rows past n are zero)
  for (int i = tid; i < kRows * (D / 4); i += kRvqThreads) {
    const int row = i / (D / 4), c = (i % (D / 4)) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row0 + row < a.n) {
      const uint16_t* src = a.x + (row0 + row) * a.x_stride + c;
      v = make_float4(__uint_as_float((uint32_t)src[0] << 16), __uint_as_float((uint32_t)src[1] << 16),
                      __uint_as_float((uint32_t)src[2] << 16), __uint_as_float((uint32_t)src[3] << 16));
    }
    *reinterpret_cast<float4*>(R + sw_off(row, c, kRows)) = v;
  }
  tc::fence_proxy_async_smem();  // residual visible to the MMA's operand reads
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  const int erow = 32 * (warp & 3) + lane;  // epilogue: TMEM lane quarter = warp % 4
  const bool has_row = warp >= 1 && row0 + erow < a.n;
  const uint32_t idesc = idesc_tf32_f32(kRows, M);
  int stage_done = 0;  // stages whose copies and MMAs have landed (thread 0's view)
  int cb_issued = 0, mma_issued = 0;  // thread 0: codebook copies / MMA batches issued

  for (int s = 0; s < a.S; ++s) {
    // ---- codebook of stage s -> C (TMA), then ||C_s[m]||^2 and max ||C_s[m]||
    if (tid == 0) {
      tc::mbar_arrive_expect_tx(&bars->cb_full, (uint32_t)(L::kBlocks * M * 128));
      for (int blk = 0; blk < L::kBlocks; ++blk)
        tc::tma_load_2d(C + (size_t)blk * M * 128, &cmap, &bars->cb_full, blk * 32, s * M);
      cb_issued = s + 1;
    }
    const bool got = tc::mbar_wait(&bars->cb_full, s & 1, &bars->abort);
    if (__syncthreads_or(!got)) break;
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
    if (tid == 0) bars->cmax = 0.f;
    __syncthreads();
    if (lane == 0) atomicMax(reinterpret_cast<int*>(&bars->cmax), __float_as_int(my_max));  // >= 0: int order
    // ---- scores: TMEM[row][m] = r . C_s[m] (tf32), 8 elements per K-step
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
    const bool scored = tc::mbar_wait(&bars->mma_done, s & 1, &bars->abort);
    if (__syncthreads_or(!scored)) break;
    if (tid == 0) stage_done = s + 1;
    tc::tc_fence_after();
    const float cmax = sqrtf(bars->cmax);

    // ---- decision: approximate best, then exact fp32 distances of the candidates
    if (warp >= 1) {
      float rr = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; c += 4) {
        const float4 v = *reinterpret_cast<const float4*>(R + sw_off(erow, c, kRows));
        rr = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, rr))));
      }
      // tf32 keeps 10 mantissa bits of each operand, so with the fp32 sums
      // |r.c - (MMA dot)| < 2^-8.9 ||r|| ||c|| and |||c||^2 - cnorm| < 2^-17
      // cmax^2 (d <= 128 terms).  Two approximate scores therefore differ from
      // the exact difference of the distances by less than
      // 2^-6.9 ||r|| cmax + 2^-16 cmax^2: every codeword within that band of
      // the best approximate score is a candidate, and the exact argmin is
      // always among them
      const float band = 0x1p-6f * sqrtf(rr) * cmax + 0x1p-15f * (rr + cmax * cmax) + 1e-30f;
      const uint32_t base = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
      float best = INFINITY;
      for (int c0 = 0; c0 < M; c0 += 32) {
        uint32_t x[32];
        KVC_TMEM_LD32(base + (uint32_t)c0, x);
        KVC_TMEM_WAIT_LD32(x);
        const int ncol = M - c0;  // 16 or >= 32 (M % 16 == 0): columns past M hold no score
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (e < ncol) best = fminf(best, cnorm[c0 + e] - 2.f * __uint_as_float(x[e]));
      }
      const float limit = best + band;
      float exact_best = INFINITY;
      int arg = 0;
      for (int c0 = 0; c0 < M; c0 += 32) {
        uint32_t x[32];
        KVC_TMEM_LD32(base + (uint32_t)c0, x);
        KVC_TMEM_WAIT_LD32(x);
        uint32_t cand = 0;  // candidates of this group of 32 codewords, one bit each
        const int ncol = M - c0;
#pragma unroll
        for (int e = 0; e < 32; ++e)
          cand |= (e < ncol && cnorm[c0 + e] - 2.f * __uint_as_float(x[e]) <= limit ? 1u : 0u) << e;
        while (cand) {
          const int m = c0 + __ffs(cand) - 1;  // ascending m
          cand &= cand - 1;
          float dist = 0.f;
#pragma unroll 8
          for (int c = 0; c < D; c += 4) {
            const float4 rv = *reinterpret_cast<const float4*>(R + sw_off(erow, c, kRows));
            const float4 cv = *reinterpret_cast<const float4*>(C + sw_off(m, c, M));
            const float d0 = rv.x - cv.x, d1 = rv.y - cv.y, d2 = rv.z - cv.z, d3 = rv.w - cv.w;
            dist = fmaf(d0, d0, fmaf(d1, d1, fmaf(d2, d2, fmaf(d3, d3, dist))));
          }
          if (dist < exact_best) {  // ascending m: ties keep the lowest index
            exact_best = dist;
            arg = m;
          }
        }
        __syncwarp();
      }
      if (has_row) a.codes[(row0 + erow) * a.S + s] = arg;
      // residual update (rows past n keep their zeros: code 0 is harmless)
      if (has_row) {
#pragma unroll 8
        for (int c = 0; c < D; c += 4) {
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
