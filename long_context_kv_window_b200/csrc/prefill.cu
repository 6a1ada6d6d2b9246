// prefill.cu -- causal prefill attention with each query row's log-sum-exp, on tcgen05.
//
// FastKV (gist.science 2502.01068) section 1: during prefill every layer runs
// full causal attention over the prompt; section 2.A: at the TSP layer that
// attention covers the whole prompt, so the log-sum-exp of the observation
// window's rows -- the softmax normalisers of the token scores -- comes out of
// it (kvc_score_lse consumes them and reads K once).  FastKV abstract:
// grouped-query heads (query head h reads KV head h / G).  The same kernel is
// the attention of the later layers over the TSP-propagated tokens (their
// positions ascend, so causality carries over to the compacted sequence).
//
// CTA (query block of 128 rows, query head h), key tiles of 128 up to the
// diagonal:
//   S = Q_blk . K_t^T   tcgen05 kind::f16, M = 128 queries, N = 128 keys,
//                       K = d = 128, fp32 in TMEM (two buffers);
//   P = 2^(S*c - m)     one thread per query row (TMEM lane), c = scale*log2 e,
//                       m the row's running reference, P as bf16 in shared
//                       memory (two buffers, the A operand);
//   O += P . V_t        M = 128 queries, N = d = 128, K = 128 keys, the V tile
//                       as the TMA wrote it read as an MN-major B operand, O in
//                       TMEM across the key tiles.
// The reference moves only when a row's max passes it by more than 8 log2
// units (p <= 2^8 otherwise, carried exactly enough by bf16 and fp32): then
// the warp waits for the last output MMA and rescales its rows of O in TMEM.
// The row sums are kept twice: over the bf16 P (the normaliser of O, so the
// output is a convex combination of V rows) and, in fp64 across tiles, over
// the fp32 p (the log-sum-exp, which the token scores need to ~1e-6).
//
// Warp roles: 0 Q and K producer, 1 TMEM allocator + MMA issuer, 2..5 softmax
// (TMEM lane quarter = warp & 3), 6 V producer.  Every wait is bounded; on a
// timeout the CTA records KVC_DEV_ERR_TIMEOUT, lets its copies and MMAs land,
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

constexpr int kPT = 128;             // queries per block, keys per tile
constexpr int kPBlock = 224;         // 7 warps
constexpr uint32_t kPCols = 512;     // S: 2 x 128 columns, O: 128
constexpr uint32_t kPO = 256;        // first O column
constexpr float kPSlack = 8.f;       // log2 units a row max may pass its reference by
constexpr double kLn2 = 0.6931471805599453;
constexpr double kLog2e = 1.4426950408889634;

struct PreArgs {
  int64_t n;
  int H, Hkv, G;
  float c;           // scale * log2(e)
  uint16_t* out;     // [n][H][128] bf16 or nullptr
  float* lse;        // [n][H] or nullptr
  int32_t* err;
};

struct PreSmem {
  static constexpr int kBlk = kPT * 128;          // 128 rows x 128 B: one 64-column block (16 KB)
  static constexpr int kTile = 2 * kBlk;          // a 128 x 128 bf16 tile (32 KB)
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kTile;     // K ring, 2 tiles
  static constexpr int kVOff = kKOff + 2 * kTile; // V ring, 2 tiles
  static constexpr int kPOff = kVOff + 2 * kTile; // P, 2 buffers
  static constexpr int kBarOff = kPOff + 2 * kTile;
  static constexpr size_t kBytes = 1024 + (size_t)kBarOff + 1024;
};

struct PreBars {
  uint64_t qfull;
  uint64_t kfull[2], kempty[2], vfull[2], vempty[2];
  uint64_t s_full[2], s_empty[2], p_full[2], o_done[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

// 32 lanes x 32 fp32 columns back into TMEM, and the wait for this thread's stores.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// MN-major operand descriptor, 128-byte swizzle: 64 MN-consecutive elements
// per 128-byte row, K rows at 128 B; `lbo` bytes between 64-element MN
// blocks, 1024 B between 8-row K groups.
__device__ __forceinline__ uint64_t desc_mn_sw128_p(uint32_t smem_addr, uint32_t lbo) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

__global__ void __launch_bounds__(kPBlock, 1)
prefill_attention_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap vmap, const PreArgs a) {
  using L = PreSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  PreBars* bars = reinterpret_cast<PreBars*>(sm + L::kBarOff);
  static_assert(sizeof(PreBars) <= 1024, "barrier block");

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nqb = (int)((a.n + kPT - 1) / kPT);
  const int qb = nqb - 1 - (int)blockIdx.x;  // the longest rows first
  const int h = blockIdx.y, g = h / a.G;
  const int nt = qb + 1;                      // key tiles up to the diagonal

  if (tid == 0) {
    tc::mbar_init(&bars->qfull, 1);
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&bars->kfull[b], 1);
      tc::mbar_init(&bars->kempty[b], 1);
      tc::mbar_init(&bars->vfull[b], 1);
      tc::mbar_init(&bars->vempty[b], 1);
      tc::mbar_init(&bars->s_full[b], 1);
      tc::mbar_init(&bars->s_empty[b], 4);
      tc::mbar_init(&bars->p_full[b], 4);
      tc::mbar_init(&bars->o_done[b], 1);
    }
    tc::mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    tc::fence_mbar_init();
    tc::prefetch_tmap(&qmap);
    tc::prefetch_tmap(&kmap);
    tc::prefetch_tmap(&vmap);
  }
  if (warp == 1) {
    tc::tmem_alloc(&bars->tmem_base, kPCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  pdl_wait();  // q, k, v may come from the previous kernel of the stream
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;

  if (warp == 0 || warp == 6) {
    // ---- producers: warp 0 the Q block and the K tiles, warp 6 the V tiles
    if (lane == 0) {
      const bool is_k = warp == 0;
      const CUtensorMap* map = is_k ? &kmap : &vmap;
      uint64_t* fullb = is_k ? bars->kfull : bars->vfull;
      uint64_t* emptyb = is_k ? bars->kempty : bars->vempty;
      uint8_t* ring = sm + (is_k ? L::kKOff : L::kVOff);
      if (is_k) {
        tc::mbar_arrive_expect_tx(&bars->qfull, (uint32_t)L::kTile);
        for (int cb = 0; cb < 2; ++cb)
          tc::tma_load_3d(sm + L::kQOff + cb * L::kBlk, &qmap, &bars->qfull, cb * 64, h, qb * kPT);
      }
      int issued = 0;
      for (int t = 0; t < nt; ++t) {
        const int b = t & 1;
        if (t >= 2 && !tc::mbar_wait(&emptyb[b], ((t >> 1) - 1) & 1, abort_flag)) break;
        tc::mbar_arrive_expect_tx(&fullb[b], (uint32_t)L::kTile);
        for (int cb = 0; cb < 2; ++cb)
          tc::tma_load_3d(ring + b * L::kTile + cb * L::kBlk, map, &fullb[b], cb * 64, g, t * kPT);
        issued = t + 1;
      }
      if (*abort_flag) {
        if (is_k) tc::mbar_drain(&bars->qfull, 0);
        for (int t = std::max(0, issued - 2); t < issued; ++t) tc::mbar_drain(&fullb[t & 1], (t >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer: the logits of tile t, then the output of tile t - 1
    if (lane == 0) {
      const uint32_t id_s = tc::idesc_bf16_f32(128, 128);
      const uint32_t id_o = tc::idesc_bf16_f32(128, 128) | (1u << 16);  // B (V) MN-major
      const uint64_t q_desc = tc::desc_k_sw128(tc::smem_u32(sm + L::kQOff));
      const uint64_t k_desc = tc::desc_k_sw128(tc::smem_u32(sm + L::kKOff));
      const uint64_t p_desc = tc::desc_k_sw128(tc::smem_u32(sm + L::kPOff));
      const uint64_t v_desc = desc_mn_sw128_p(tc::smem_u32(sm + L::kVOff), (uint32_t)L::kBlk);
      bool ok = tc::mbar_wait(&bars->qfull, 0, abort_flag);
      for (int t = 0; ok && t <= nt; ++t) {
        if (t < nt) {
          const int b = t & 1;
          ok = tc::mbar_wait(&bars->kfull[b], (t >> 1) & 1, abort_flag);
          if (ok && t >= 2) ok = tc::mbar_wait(&bars->s_empty[b], ((t >> 1) - 1) & 1, abort_flag);
          if (!ok) break;
          tc::tc_fence_after();
          const uint64_t kd = k_desc + (uint64_t)(((uint32_t)b * L::kTile) >> 4);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t off = (uint32_t)((ks >> 2) * L::kBlk + (ks & 3) * 32) >> 4;
            tc::mma_bf16(tmem + (uint32_t)(128 * b), q_desc + off, kd + off, id_s, ks != 0);
          }
          tc::mma_commit(&bars->s_full[b]);
          tc::mma_commit(&bars->kempty[b]);  // the K tile is read
        }
        if (t >= 1) {
          const int u = t - 1, b = u & 1;
          ok = tc::mbar_wait(&bars->p_full[b], (u >> 1) & 1, abort_flag);
          if (ok) ok = tc::mbar_wait(&bars->vfull[b], (u >> 1) & 1, abort_flag);
          if (!ok) break;
          tc::tc_fence_after();
          const uint64_t pd = p_desc + (uint64_t)(((uint32_t)b * L::kTile) >> 4);
          const uint64_t vd = v_desc + (uint64_t)(((uint32_t)b * L::kTile) >> 4);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t poff = (uint32_t)((ks >> 2) * L::kBlk + (ks & 3) * 32) >> 4;  // 16 keys of P
            const uint32_t voff = (uint32_t)(ks * 16 * 128) >> 4;                         // 16 V rows
            tc::mma_bf16(tmem + kPO, pd + poff, vd + voff, id_o, (u > 0 || ks > 0) ? 1u : 0u);
          }
          tc::mma_commit(&bars->o_done[b]);
          tc::mma_commit(&bars->vempty[b]);  // the V tile is read
        }
      }
      tc::mma_commit(&bars->mma_done);  // every MMA issued above has completed before TMEM is freed
      tc::mbar_drain(&bars->mma_done, 0);
    }
  } else {
    // ---- softmax: one query row per thread
    const int wq = warp & 3;
    const int r = 32 * wq + lane;
    const int64_t qi = (int64_t)qb * kPT + r;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * wq) << 16);
    uint8_t* prow = sm + L::kPOff + r * 128;  // this row in P (block 0; block 1 at + kBlk)
    float m_ref = -INFINITY, l_round = 0.f;
    double l_exact = 0.0;
    bool ok = true;
    for (int t = 0; t < nt; ++t) {
      const int b = t & 1;
      if (!tc::mbar_wait(&bars->s_full[b], (t >> 1) & 1, abort_flag)) { ok = false; break; }
      tc::tc_fence_after();
      uint32_t x[128];
      {
        uint32_t* x1 = x + 64;
        KVC_TMEM_LD64(lane_base + (uint32_t)(128 * b), x);
        KVC_TMEM_LD64(lane_base + (uint32_t)(128 * b + 64), x1);
        KVC_TMEM_WAIT_LD64(x);
        KVC_TMEM_TIE32(x1);
        uint32_t* x2 = x + 96;
        KVC_TMEM_TIE32(x2);
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars->s_empty[b]);
      // the diagonal tile: key t*128 + c is visible to row r when c <= r
      const int lim = (t == nt - 1) ? r : kPT - 1;
      if (t == nt - 1) {
#pragma unroll
        for (int e = 0; e < kPT; ++e)
          if (e > lim) x[e] = __float_as_uint(-INFINITY);
      }
      float mx = -INFINITY;
#pragma unroll
      for (int e = 0; e < kPT; ++e) mx = fmaxf(mx, __uint_as_float(x[e]));
      const float mc = mx * a.c;
      const bool move = m_ref == -INFINITY || mc > m_ref + kPSlack;
      float alpha = 1.f;
      if (move) {
        alpha = m_ref == -INFINITY ? 0.f : tc::ex2_approx(m_ref - mc);
        l_round *= alpha;
        l_exact *= (double)alpha;
        m_ref = mc;
      }
      // O rows of this warp rescaled in TMEM once the last output MMA is done
      if (t > 0 && __any_sync(0xffffffffu, move)) {
        const int u = t - 1;
        if (!tc::mbar_wait(&bars->o_done[u & 1], (u >> 1) & 1, abort_flag)) { ok = false; break; }
        tc::tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t o[32];
          KVC_TMEM_LD32(lane_base + kPO + (uint32_t)c0, o);
          KVC_TMEM_WAIT_LD32(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(lane_base + kPO + (uint32_t)c0, o);
        }
        tmem_wait_st();
      }
      // P buffer b was last read by the output MMA of tile t - 2
      if (t >= 2 && !tc::mbar_wait(&bars->o_done[b], ((t >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
      // p in packed pairs, its bf16 copy into P, and both row sums on two
      // accumulators each (short dependency chains)
      const float2 c2 = make_float2(a.c, a.c), nm2 = make_float2(-m_ref, -m_ref);
      float2 se2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      float2 sr2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      uint8_t* pb = prow + b * L::kTile;
#pragma unroll
      for (int c8 = 0; c8 < kPT; c8 += 8) {
        uint32_t w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 t2 =
              tc::fma2(make_float2(__uint_as_float(x[c8 + 2 * u]), __uint_as_float(x[c8 + 2 * u + 1])), c2, nm2);
          const float2 p2 = make_float2(tc::ex2_approx(t2.x), tc::ex2_approx(t2.y));
          const __nv_bfloat162 hp = __floats2bfloat162_rn(p2.x, p2.y);
          se2[u & 1] = tc::add2(se2[u & 1], p2);
          sr2[u & 1] = tc::add2(sr2[u & 1], __bfloat1622float2(hp));
          w[u] = *reinterpret_cast<const uint32_t*>(&hp);
        }
        const int blk = c8 >> 6, ch = ((c8 & 63) >> 3) ^ (r & 7);
        *reinterpret_cast<uint4*>(pb + blk * L::kBlk + (ch << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      const float2 se = tc::add2(se2[0], se2[1]), sr = tc::add2(sr2[0], sr2[1]);
      l_round += sr.x + sr.y;
      l_exact += (double)(se.x + se.y);
      tc::fence_proxy_async_smem();  // P visible to the tensor core
      tc::tc_fence_before();         // (and the O rescale stores)
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars->p_full[b]);
    }
    // ---- the output rows and log-sum-exp
    if (ok) {
      const int u = nt - 1;
      ok = tc::mbar_wait(&bars->o_done[u & 1], (u >> 1) & 1, abort_flag);
    }
    if (ok) {
      tc::tc_fence_after();
      const bool store = qi < a.n;
      const float inv = 1.f / l_round;
#pragma unroll
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t o[32];
        KVC_TMEM_LD32(lane_base + kPO + (uint32_t)c0, o);
        KVC_TMEM_WAIT_LD32(o);
        if (store && a.out) {
          uint4* dst = reinterpret_cast<uint4*>(a.out + (qi * a.H + h) * 128 + c0);
#pragma unroll
          for (int v8 = 0; v8 < 4; ++v8) {
            uint32_t w[4];
#pragma unroll
            for (int u2 = 0; u2 < 4; ++u2) {
              const __nv_bfloat162 hp = __floats2bfloat162_rn(__uint_as_float(o[8 * v8 + 2 * u2]) * inv,
                                                              __uint_as_float(o[8 * v8 + 2 * u2 + 1]) * inv);
              w[u2] = *reinterpret_cast<const uint32_t*>(&hp);
            }
            dst[v8] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      if (store && a.lse) a.lse[qi * a.H + h] = (float)(((double)m_ref + log2(l_exact)) * kLn2);
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (*abort_flag && tid == 0) set_dev_err(a.err, KVC_DEV_ERR_TIMEOUT);
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kPCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D map over a [n][heads][128] bf16 tensor: boxes of 64 columns x 1 head x 128 rows.
kvc_status make_map(CUtensorMap* m, const uint16_t* base, int heads, int64_t n) {
  cuuint64_t dims[3] = {128u, (cuuint64_t)heads, (cuuint64_t)n};
  cuuint64_t strides[2] = {(cuuint64_t)128 * 2, (cuuint64_t)heads * 128 * 2};
  cuuint32_t box[3] = {64u, 1u, (cuuint32_t)kPT};
  cuuint32_t es[3] = {1u, 1u, 1u};
  if (heads == 1) strides[0] = strides[1];  // a size-1 dim still needs a legal stride
  if (encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return fail(KVC_ERR_CUDA, "cuTensorMapEncodeTiled failed for the prefill operands");
  return KVC_OK;
}

}  // namespace
}  // namespace kvc

using namespace kvc;

extern "C" kvc_status kvc_prefill_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t n,
                                            int32_t num_heads, int32_t num_kv_heads, int32_t head_dim, float scale,
                                            uint16_t* out, float* lse, int32_t* dev_err, void* stream) {
  clear_error();
  KVC_CHECK_ARG(q && k && v, "q, k and v must be non-NULL");
  if (head_dim != 128) return fail(KVC_ERR_UNSUPPORTED, "head_dim must be 128");
  KVC_CHECK_ARG(num_heads >= 1 && num_kv_heads >= 1 && num_heads % num_kv_heads == 0 && num_heads <= 65535,
                "num_heads must be a positive multiple of num_kv_heads (<= 65535)");
  KVC_CHECK_ARG(n >= 1 && n < (int64_t(1) << 31), "need 1 <= n < 2^31");
  KVC_CHECK_ARG(scale > 0.f && scale < 1e30f, "scale must be positive and finite");
  KVC_CHECK_ARG(aligned(q, 16) && aligned(k, 16) && aligned(v, 16) && (!out || aligned(out, 16)),
                "q, k, v and out must be 16-byte aligned");
  if (!encode_fn()) return fail(KVC_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  CUtensorMap maps[3];
  kvc_status s = make_map(&maps[0], q, num_heads, n);
  if (s == KVC_OK) s = make_map(&maps[1], k, num_kv_heads, n);
  if (s == KVC_OK) s = make_map(&maps[2], v, num_kv_heads, n);
  if (s != KVC_OK) return s;
  PreArgs a{};
  a.n = n;
  a.H = num_heads;
  a.Hkv = num_kv_heads;
  a.G = num_heads / num_kv_heads;
  a.c = (float)((double)scale * kLog2e);
  a.out = out;
  a.lse = lse;
  a.err = dev_err;
  static ContextCache cache;
  s = once_per_context(cache, [] {
    KVC_CUDA_TRY(cudaFuncSetAttribute(prefill_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)PreSmem::kBytes));
    return KVC_OK;
  });
  if (s != KVC_OK) return s;
  const unsigned nqb = (unsigned)((n + kPT - 1) / kPT);
  const Launch l(dim3(nqb, (unsigned)num_heads), dim3(kPBlock), PreSmem::kBytes, (cudaStream_t)stream);
  KVC_CUDA_TRY(l.run(prefill_attention_kernel, maps[0], maps[1], maps[2], a));
  count_launch();
  return KVC_OK;
}
