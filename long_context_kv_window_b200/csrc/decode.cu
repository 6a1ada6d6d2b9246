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

// Chunks per KV head: about two CTAs per SM in all, never more than one per tile.
int decode_chunks(int64_t kk, int Hkv) {
  const int64_t tiles = (kk + kT - 1) / kT;
  const int64_t want = std::min<int64_t>(kMaxChunks, std::max<int64_t>(1, kDecCtaTarget / Hkv));
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
