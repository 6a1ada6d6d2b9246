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
// second kernel merges the partials of each head.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "tc.cuh"

namespace kvc {
namespace {

constexpr int kT = 64;             // retained entries per tile
constexpr int kDecThreads = 256;
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
  float* out;         // [H][d]
  int32_t* err;
};

template <int D>
struct DecSmem {
  static constexpr int kBoxes = D / 64;                      // 64-element (128-byte) column blocks
  static constexpr int kMatBytes = kBoxes * kT * 128;        // one K or V tile
  static constexpr int kStageBytes = 2 * kMatBytes;          // K tile, then V tile
  static constexpr size_t kFloats = (size_t)kDecMaxG * (D + 16) + (size_t)kDecMaxG * kT + 3 * kDecMaxG;
  static_assert((size_t)kDecStages * kStageBytes >= (size_t)(kDecThreads / (D / 2)) * kDecMaxG * D * 4,
                "the partial reduction reuses the stages");
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
template <int D, int KG>
__global__ void __launch_bounds__(kDecThreads, 2)
decode_partial_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                      const DecArgs a) {
  using L = DecSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stages = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* qs = reinterpret_cast<float*>(stages + (size_t)kDecStages * L::kStageBytes);  // [KG][D + 16]
  float* P = qs + kDecMaxG * (D + 16);                                                  // [kT][KG]: logits, then p
  float* m_run = P + kDecMaxG * kT;
  float* l_run = m_run + kDecMaxG;
  float* alpha = l_run + kDecMaxG;
  uint64_t* full = reinterpret_cast<uint64_t*>((reinterpret_cast<uintptr_t>(alpha + kDecMaxG) + 15) & ~uintptr_t(15));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + kDecStages);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.y, chunk = blockIdx.x;
  const int G = a.G;
  constexpr int kQuarter = D / 4;            // dimensions per logit thread
  constexpr int kQRow = D + 16;              // floats per head of q (four padded quarters)
  const int64_t e0 = (int64_t)chunk * a.chunk;
  const int64_t e1 = std::min<int64_t>(a.kk, e0 + a.chunk);
  const int ntiles = (int)((e1 - e0 + kT - 1) / kT);
  const int64_t row0 = (int64_t)g * a.kk + e0;  // first row of the chunk in the [Hkv*kk][D] view

  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) tc::mbar_init(&full[s], 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
    tc::prefetch_tmap(&kmap);
    tc::prefetch_tmap(&vmap);
  }
  if (tid < kDecMaxG) {
    m_run[tid] = -INFINITY;
    l_run[tid] = 0.f;
  }
  pdl_wait();  // Kc / Vc / q may come from the previous kernel of the stream
  // q as fp32, each head's D values in four quarters of D/4, every quarter
  // padded by 4 floats: the four threads of an entry read their quarters at
  // different shared-memory banks
  for (int i = tid; i < KG * D; i += kDecThreads) {
    const int h = i / D, e = i % D;
    qs[h * kQRow + (e / kQuarter) * (kQuarter + 4) + e % kQuarter] =
        h < G ? __uint_as_float((uint32_t)a.q[(int64_t)(g * G + h) * a.q_sh + e] << 16) : 0.f;
  }
  __syncthreads();

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
  int issued = 0;  // thread 0
  if (tid == 0)
    for (; issued < min(ntiles, kDecStages); ++issued) issue(issued);

  // Logits: four threads per entry, each a quarter of the D dimensions for
  // every head of the group (one read and unpack of each K element).
  constexpr int kQChunks = kQuarter / 8;     // 16-byte chunks per thread
  const int lj = tid >> 2, lq = tid & 3;     // entry, quarter
  // Output: one thread per pair of dimensions and group of entries; it adds
  // every head's p * v for its entries (one read of each V element).
  constexpr int kPairs = D / 2;
  constexpr int kGroups = kDecThreads / kPairs;  // 4 (D = 128) or 8 (D = 64)
  constexpr int kPerGroup = kT / kGroups;
  const int dp = tid % kPairs, og = tid / kPairs;
  const int oe = 2 * dp, ocb = oe / 64, oe64 = oe % 64;
  float2 o[KG];
#pragma unroll
  for (int h = 0; h < KG; ++h) o[h] = make_float2(0.f, 0.f);

  int t = 0;
  for (; t < ntiles; ++t) {
    const int s = t % kDecStages;
    const bool ok = tc::mbar_wait(&full[s], (t / kDecStages) & 1, abort_flag);
    if (__syncthreads_or(!ok)) break;  // every thread leaves together
    const uint8_t* kt = stages + (size_t)s * L::kStageBytes;
    const uint8_t* vt = kt + L::kMatBytes;
    const int nvalid = (int)std::min<int64_t>(kT, e1 - (e0 + (int64_t)t * kT));

    // ---- logits (log2 domain), entry-major P[j][h]
    {
      float2 acc[KG];
#pragma unroll
      for (int h = 0; h < KG; ++h) acc[h] = make_float2(0.f, 0.f);
      if (lj < nvalid) {
#pragma unroll
        for (int c = 0; c < kQChunks; ++c) {
          const int col = lq * kQuarter + c * 8;  // first dimension of this chunk
          const int cb = col / 64, k16 = (col % 64) / 8;
          const uint4 kw = *reinterpret_cast<const uint4*>(kt + cb * kT * 128 + sw128(lj, k16));
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
      }
#pragma unroll
      for (int h = 0; h < KG; ++h) {
        float v = acc[h].x + acc[h].y;
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        if (lq == 0) P[lj * KG + h] = lj < nvalid ? v * a.c : -INFINITY;
      }
    }
    __syncthreads();

    // ---- online softmax per head: one warp per head
    for (int h = warp; h < G; h += kDecThreads / 32) {
      const float x0 = P[lane * KG + h], x1 = P[(lane + 32) * KG + h];
      float mx = fmaxf(x0, x1);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_old = m_run[h];
      const float m_new = fmaxf(m_old, mx);
      float p0 = 0.f, p1 = 0.f;
      if (m_new != -INFINITY) {
        p0 = tc::ex2_approx(x0 - m_new);
        p1 = tc::ex2_approx(x1 - m_new);
      }
      P[lane * KG + h] = p0;
      P[(lane + 32) * KG + h] = p1;
      float sum = p0 + p1;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      if (lane == 0) {
        const float al = (m_old == -INFINITY) ? 0.f : tc::ex2_approx(m_old - m_new);
        l_run[h] = l_run[h] * al + sum;
        m_run[h] = m_new;
        alpha[h] = al;
      }
    }
    __syncthreads();

    // ---- output rows: o_h <- alpha_h * o_h + sum_j p_hj v_j (this thread's
    // two dimensions, its group of entries; masked entries have p = 0, and
    // their V rows are real data or TMA zero fill)
    {
#pragma unroll
      for (int h = 0; h < KG; ++h) {
        const float al = h < G ? alpha[h] : 0.f;
        o[h] = make_float2(o[h].x * al, o[h].y * al);
      }
      const uint8_t* vcol = vt + ocb * kT * 128 + (oe64 & 7) * 2;
      const int k16 = oe64 >> 3;
      const int jb = og * kPerGroup, je = min(nvalid, jb + kPerGroup);
      for (int j = jb; j < je; ++j) {
        const float2 v = bf16x2_to_f2(*reinterpret_cast<const uint32_t*>(vcol + sw128(j, k16)));
        const float* pj = P + j * KG;
#pragma unroll
        for (int h = 0; h < KG; ++h) o[h] = tc::fma2(v, make_float2(pj[h], pj[h]), o[h]);
      }
    }
    __syncthreads();  // stage s and P are free
    if (tid == 0 && issued < ntiles) issue(issued++);
  }

  if (*abort_flag) {
    if (tid == 0) {
      // let every copy already issued land before shared memory is released
      for (int u = t; u < issued; ++u) tc::mbar_drain(&full[u % kDecStages], (u / kDecStages) & 1);
      set_dev_err(a.err, KVC_DEV_ERR_TIMEOUT);
    }
    return;
  }
  // ---- this chunk's partial: sum the entry groups of every (head, pair)
  // through shared memory (the stages are free now), then write
  float* red = reinterpret_cast<float*>(stages);  // [kGroups][G][D]
#pragma unroll
  for (int h = 0; h < KG; ++h)
    if (h < G) *reinterpret_cast<float2*>(red + ((size_t)og * G + h) * D + oe) = o[h];
  __syncthreads();
  for (int i = tid; i < G * D; i += kDecThreads) {
    float sum = 0.f;
    for (int q = 0; q < kGroups; ++q) sum += red[(size_t)q * G * D + i];
    const int h = i / D, e = i % D;
    a.part_o[((size_t)(g * G + h) * a.nchunks + chunk) * D + e] = sum;
  }
  if (tid < G) {
    a.part_m[(size_t)(g * G + tid) * a.nchunks + chunk] = m_run[tid];
    a.part_l[(size_t)(g * G + tid) * a.nchunks + chunk] = l_run[tid];
  }
}

// Merge the chunk partials of head h: out = sum_c 2^(m_c - M) o_c / sum_c 2^(m_c - M) l_c.
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const DecArgs a) {
  pdl_wait();
  const int h = blockIdx.x, e = threadIdx.x;
  const float* pm = a.part_m + (size_t)h * a.nchunks;
  const float* pl = a.part_l + (size_t)h * a.nchunks;
  float M = -INFINITY;
  for (int c = 0; c < a.nchunks; ++c) M = fmaxf(M, pm[c]);
  float L = 0.f, O = 0.f;
  for (int c = 0; c < a.nchunks; ++c) {
    if (pm[c] == -INFINITY) continue;
    const float w = tc::ex2_approx(pm[c] - M);
    L += w * pl[c];
    O += w * a.part_o[((size_t)h * a.nchunks + c) * D + e];
  }
  a.out[(size_t)h * D + e] = O / L;
}

// Chunks per KV head: about two CTAs per SM in all, never more than one per tile.
int decode_chunks(int64_t kk, int Hkv) {
  const int64_t tiles = (kk + kT - 1) / kT;
  const int64_t want = std::max<int64_t>(1, kDecCtaTarget / Hkv);
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
  const size_t nch = (size_t)decode_chunks(kk, Hkv);
  return round_up((size_t)H * nch * 4, kWsAlign) * 2 + round_up((size_t)H * nch * d * 4, kWsAlign);
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
  KVC_CHECK_ARG(aligned(k_c, 16) && aligned(v_c, 16), "k_c and v_c must be 16-byte aligned");
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
  const int d = head_dim, Hkv = num_kv_heads;
  CUtensorMap maps[2];
  const uint16_t* srcs[2] = {k_c, v_c};
  for (int i = 0; i < 2; ++i) {
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)(kk * Hkv)};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {64u, (cuuint32_t)kT};
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
  a.nchunks = decode_chunks(kk, Hkv);
  const int64_t tiles = (kk + kT - 1) / kT;
  a.chunk = (int)(((tiles + a.nchunks - 1) / a.nchunks) * kT);
  a.c = (float)((double)scale * kLog2e);
  WsCursor wc{static_cast<char*>(ws), ws_bytes};
  a.part_m = wc.take<float>((size_t)num_heads * a.nchunks);
  a.part_l = wc.take<float>((size_t)num_heads * a.nchunks);
  a.part_o = wc.take<float>((size_t)num_heads * a.nchunks * d);
  if (!wc.ok) return fail(KVC_ERR_WORKSPACE, "decode workspace too small");
  a.out = out;
  a.err = dev_err;

  const int kg = decode_group_slots(a.G);
  const cudaStream_t st = (cudaStream_t)stream;
  {
    const size_t smem = d == 128 ? DecSmem<128>::kBytes : DecSmem<64>::kBytes;
    const Launch l(dim3((unsigned)a.nchunks, (unsigned)Hkv), dim3(kDecThreads), smem, st);
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
