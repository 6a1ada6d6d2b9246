// gather.cu -- compaction of retained K/V rows and of propagated hidden states.
//
// FastKV (gist.science 2502.01068) section 2.B: the KV entries retained per
// layer form the compacted cache used at decode; section 2.A: after the TSP
// layer only the selected tokens' hidden states (window included) go on.
// FastKV abstract: the retained set is per KV head (GQA-aware).
//
// Both kernels are pure bit copies bound by HBM bandwidth: 16-byte vector
// loads/stores, several loads in flight per thread before the first store,
// streaming (evict-first) stores for the outputs that are written once.
#include "common.cuh"

namespace kvc {
namespace {

constexpr int kGatherThreads = 256;
constexpr int kKvUnroll = 4;   // uint4 items per thread per iteration (x2 with V)
constexpr int kHidUnroll = 8;  // uint4 per lane in flight (hidden rows)

// Vectors of 16 B per head row: D/8 (8 for d=64, 16 for d=128).
template <int VPR>
__global__ void __launch_bounds__(kGatherThreads)
gather_kv_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, int64_t sn, int64_t sh,
                 const int32_t* __restrict__ cu, int64_t n, int Hkv, const int32_t* __restrict__ idx,
                 int64_t idx_row_stride, int64_t kk, uint4* __restrict__ k_out,
                 uint4* __restrict__ v_out, int32_t* err) {
  pdl_wait();
  // blockIdx.y = b * Hkv + g ; blockIdx.x covers kk * VPR items of that head
  const int bg = blockIdx.y;
  const int g = bg % Hkv;
  const int b = bg / Hkv;
  SeqSpan span = seq_span(cu, b, n);
  // a malformed cu_seqlens entry (negative start or length, or a sequence
  // past the packed total) gathers nothing: its rows are zero and the
  // sequence error bit is set instead of reading outside K / V
  const bool bad_span = cu != nullptr && (span.start < 0 || span.len < 0 || span.start + span.len > n);
  if (bad_span) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_dev_err(err, KVC_DEV_ERR_SEQLENS);
    span.len = 0;
  }
  const int32_t* irow = idx + (cu ? (int64_t)bg * kk : (int64_t)g * idx_row_stride);
  const int64_t items = kk * VPR;
  const int64_t out_base = (int64_t)bg * kk * VPR;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);

  for (int64_t base = (int64_t)blockIdx.x * kGatherThreads * kKvUnroll + threadIdx.x; base < items;
       base += (int64_t)gridDim.x * kGatherThreads * kKvUnroll) {
    uint4 kr[kKvUnroll], vr[kKvUnroll];
#pragma unroll
    for (int u = 0; u < kKvUnroll; ++u) {
      const int64_t it = base + (int64_t)u * kGatherThreads;
      kr[u] = zero;
      vr[u] = zero;
      if (it < items) {
        const int64_t r = it / VPR;
        const int vec = (int)(it % VPR);
        const int64_t j = irow[r];
        if (j >= 0 && j < span.len) {
          const int64_t src = (span.start + j) * sn + (int64_t)g * sh + vec;
          kr[u] = __ldg(k + src);
          if (v) vr[u] = __ldg(v + src);
        } else if (j != -1 && vec == 0 && !bad_span) {
          set_dev_err(err, KVC_DEV_ERR_INDEX);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kKvUnroll; ++u) {
      const int64_t it = base + (int64_t)u * kGatherThreads;
      if (it < items) {
        __stcs(k_out + out_base + it, kr[u]);
        if (v_out) __stcs(v_out + out_base + it, vr[u]);
      }
    }
  }
}

// One warp per output row; each lane keeps kHidUnroll 16-byte loads in flight.
__global__ void __launch_bounds__(kGatherThreads)
gather_hidden_kernel(const uint4* __restrict__ x, int64_t sn_v, int64_t n, int64_t vpr,
                     const int32_t* __restrict__ idx, int64_t kk, uint4* __restrict__ out,
                     int32_t* err) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (kGatherThreads / 32);
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  for (int64_t r = (int64_t)blockIdx.x * (kGatherThreads / 32) + (threadIdx.x >> 5); r < kk;
       r += warps) {
    const int64_t j = idx[r];
    const bool valid = (j >= 0 && j < n);
    if (!valid && j != -1 && lane == 0) set_dev_err(err, KVC_DEV_ERR_INDEX);
    const uint4* src = x + (valid ? j : 0) * sn_v;
    uint4* dst = out + r * vpr;
    for (int64_t c0 = 0; c0 < vpr; c0 += 32 * kHidUnroll) {
      uint4 t[kHidUnroll];
#pragma unroll
      for (int u = 0; u < kHidUnroll; ++u) {
        const int64_t c = c0 + u * 32 + lane;
        t[u] = (valid && c < vpr) ? __ldcs(src + c) : zero;
      }
#pragma unroll
      for (int u = 0; u < kHidUnroll; ++u) {
        const int64_t c = c0 + u * 32 + lane;
        if (c < vpr) __stcs(dst + c, t[u]);
      }
    }
  }
}

kvc_status launch_gather_kv(const uint16_t* k, const uint16_t* v, int64_t sn, int64_t sh,
                            const int32_t* cu, int32_t B, int64_t n, int32_t Hkv, int32_t d,
                            const int32_t* idx, int64_t idx_row_stride, int64_t kk,
                            uint16_t* k_out, uint16_t* v_out, int32_t* err, cudaStream_t st) {
  if (kk == 0) return KVC_OK;
  const int vpr = d / 8;
  const int64_t items = kk * vpr;
  const int64_t per_block = (int64_t)kGatherThreads * kKvUnroll;
  int64_t bx = (items + per_block - 1) / per_block;
  // enough blocks to fill the GPU several times over, grid-stride beyond that
  const int64_t cap = (int64_t)num_sms() * 16;
  if (bx * B * Hkv > cap) bx = std::max<int64_t>(1, cap / ((int64_t)B * Hkv));
  dim3 grid((unsigned)bx, (unsigned)(B * Hkv));
  auto kp = reinterpret_cast<const uint4*>(k);
  auto vp = reinterpret_cast<const uint4*>(v);
  auto ko = reinterpret_cast<uint4*>(k_out);
  auto vo = reinterpret_cast<uint4*>(v_out);
  const Launch l(grid, dim3(kGatherThreads), 0, st);
  const int64_t sn8 = sn / 8, sh8 = sh / 8;
  if (vpr == 16)
    KVC_CUDA_TRY(l.run(gather_kv_kernel<16>, kp, vp, sn8, sh8, cu, n, Hkv, idx, idx_row_stride, kk, ko, vo, err));
  else
    KVC_CUDA_TRY(l.run(gather_kv_kernel<8>, kp, vp, sn8, sh8, cu, n, Hkv, idx, idx_row_stride, kk, ko, vo, err));
  count_launch();
  return KVC_OK;
}

kvc_status check_kv_args(const uint16_t* k, const uint16_t* v, int64_t sn, int64_t sh,
                         int32_t Hkv, int32_t d, const int32_t* idx, int64_t kk,
                         const uint16_t* k_out, const uint16_t* v_out) {
  KVC_CHECK_ARG(k && idx && k_out, "k, idx and k_out must be non-NULL");
  KVC_CHECK_ARG((v == nullptr) == (v_out == nullptr), "v and v_out must both be given or both NULL");
  if (d != 64 && d != 128) return fail(KVC_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  KVC_CHECK_ARG(Hkv >= 1 && Hkv <= 65535, "num_kv_heads out of range");
  KVC_CHECK_ARG(kk >= 0 && kk * (int64_t)Hkv < (int64_t(1) << 31), "kk out of range");
  KVC_CHECK_ARG(sn % 8 == 0 && sh % 8 == 0 && sn >= 0 && sh >= 0,
                "strides must be non-negative multiples of 8 elements");
  KVC_CHECK_ARG(aligned(k, 16) && aligned(k_out, 16) && (!v || aligned(v, 16)) &&
                    (!v_out || aligned(v_out, 16)),
                "k, v, k_out, v_out must be 16-byte aligned");
  return KVC_OK;
}

}  // namespace
}  // namespace kvc

using namespace kvc;

extern "C" kvc_status kvc_gather_kv(const uint16_t* k, const uint16_t* v, int64_t stride_n,
                                    int64_t stride_h, int64_t n, int32_t num_kv_heads,
                                    int32_t head_dim, const int32_t* idx, int64_t idx_row_stride,
                                    int64_t kk, uint16_t* k_out, uint16_t* v_out, int32_t* dev_err,
                                    void* stream) {
  clear_error();
  kvc_status s = check_kv_args(k, v, stride_n, stride_h, num_kv_heads, head_dim, idx, kk, k_out, v_out);
  if (s != KVC_OK) return s;
  KVC_CHECK_ARG(n >= 0 && n < (int64_t(1) << 31), "n out of range");
  KVC_CHECK_ARG(idx_row_stride >= 0, "idx_row_stride must be >= 0");
  return launch_gather_kv(k, v, stride_n, stride_h, nullptr, 1, n, num_kv_heads, head_dim, idx,
                          idx_row_stride, kk, k_out, v_out, dev_err, (cudaStream_t)stream);
}

extern "C" kvc_status kvc_gather_kv_varlen(const uint16_t* k, const uint16_t* v, int64_t stride_n,
                                           int64_t stride_h, const int32_t* cu_seqlens,
                                           int32_t batch, int64_t total, int32_t num_kv_heads,
                                           int32_t head_dim, const int32_t* idx, int64_t kk,
                                           uint16_t* k_out, uint16_t* v_out, int32_t* dev_err,
                                           void* stream) {
  clear_error();
  kvc_status s = check_kv_args(k, v, stride_n, stride_h, num_kv_heads, head_dim, idx, kk, k_out, v_out);
  if (s != KVC_OK) return s;
  KVC_CHECK_ARG(cu_seqlens != nullptr, "cu_seqlens must be non-NULL");
  KVC_CHECK_ARG(batch >= 1 && (int64_t)batch * num_kv_heads <= 65535, "batch out of range");
  KVC_CHECK_ARG(total >= 0 && total < (int64_t(1) << 31), "total out of range");
  KVC_CHECK_ARG(kk * (int64_t)num_kv_heads * batch < (int64_t(1) << 31), "kk * Hkv * batch too large");
  return launch_gather_kv(k, v, stride_n, stride_h, cu_seqlens, batch, total, num_kv_heads,
                          head_dim, idx, kk, kk, k_out, v_out, dev_err, (cudaStream_t)stream);
}

extern "C" kvc_status kvc_gather_hidden(const uint16_t* x, int64_t stride_n, int64_t n,
                                        int64_t hidden, const int32_t* idx, int64_t kk,
                                        uint16_t* out, int32_t* dev_err, void* stream) {
  clear_error();
  KVC_CHECK_ARG(x && idx && out, "x, idx and out must be non-NULL");
  KVC_CHECK_ARG(hidden > 0 && hidden % 8 == 0, "hidden must be a positive multiple of 8");
  KVC_CHECK_ARG(stride_n >= hidden && stride_n % 8 == 0, "stride_n must be >= hidden and a multiple of 8");
  KVC_CHECK_ARG(n >= 0 && n < (int64_t(1) << 31) && kk >= 0 && kk < (int64_t(1) << 31),
                "n / kk out of range");
  KVC_CHECK_ARG(aligned(x, 16) && aligned(out, 16), "x and out must be 16-byte aligned");
  if (kk == 0) return KVC_OK;
  const int warps_per_block = kGatherThreads / 32;
  int64_t blocks = (kk + warps_per_block - 1) / warps_per_block;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  const Launch l(dim3((unsigned)blocks), dim3(kGatherThreads), 0, (cudaStream_t)stream);
  KVC_CUDA_TRY(l.run(gather_hidden_kernel, reinterpret_cast<const uint4*>(x), stride_n / 8, n, hidden / 8, idx, kk,
                     reinterpret_cast<uint4*>(out), dev_err));
  count_launch();
  return KVC_OK;
}
