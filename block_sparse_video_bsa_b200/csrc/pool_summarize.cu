// HBM-bound passes over Q, K, V.
//
//  pool_q_kernel       one CTA per (query block, head): reads the block's
//                      128 x 128 bf16 rows once, writes its fp32 mean (qpool).
//                      On a permuted (reblocked) layout it reads the rows
//                      through the permutation and also writes them out in
//                      the new order (summarize_kernel does the same for K
//                      and V), so the layout costs no separate gather pass.
//  anchor_kernel       one CTA per head: q-bar = mean of the video query rows
//                      ("the mean of the video queries as one anchor per
//                      head", Spark-H3 page, Spark-Reweight bullet), summed
//                      from qpool * n_i in a fixed order (deterministic).
//  summarize_kernel    one CTA per (key block, head): reads the K and V rows
//                      of the block once and writes the pooled key (kpool,
//                      used by the block score) and the block's summary row
//                      k~, v~, bias (the compressed branch, Spark-Reweight
//                      bullet; mean-pooled variant as the baseline it replaces).
//
// Thread layout of the per-block kernels: 256 threads, 16 threads per token
// row (8 bf16 = one 16-byte load each), 16 rows per pass, 8 passes; every
// thread keeps its 8 rows in registers, so each byte is read from HBM once.
#include "bsa_device.cuh"
#include "bsa_kernels.h"

namespace bsa {

namespace {

constexpr int kThreads = 256;

// Rows r = g + 16*it of a block (g = tid / 16), 8 dims (tid % 16) * 8 each.
__device__ __forceinline__ void load_block_rows(const __nv_bfloat16* base, int n, int g, int c,
                                                uint4 rows[8]) {
  const uint4 zero = make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int r = g + 16 * it;
    rows[it] = (r < n) ? ld_stream_v4(base + static_cast<size_t>(r) * kDim + c * 8) : zero;
  }
}

// The same rows on a permuted layout: row r of the block is row perm[row0 + r]
// of the head (clamped into the head), and each loaded chunk is also stored
// at row row0 + r of `out` (the permuted copy the attention reads).
__device__ __forceinline__ void load_block_rows_perm(const __nv_bfloat16* head,
                                                     const int32_t* perm_head, int row0, int n,
                                                     int N, int g, int c, uint4 rows[8],
                                                     __nv_bfloat16* out_head) {
  const uint4 zero = make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int r = g + 16 * it;
    if (r < n) {
      const int src = min(max(__ldg(perm_head + row0 + r), 0), N - 1);
      rows[it] = ld_stream_v4(head + static_cast<size_t>(src) * kDim + c * 8);
    } else {
      rows[it] = zero;
    }
  }
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int r = g + 16 * it;
    if (r < n)
      *reinterpret_cast<uint4*>(out_head + static_cast<size_t>(row0 + r) * kDim + c * 8) = rows[it];
  }
}

// Sum of 8-float vectors over the 16 row groups of the CTA.  Each thread
// passes its partial for dims [8c, 8c+8); thread d < 128 gets dim d's total.
// `red` is [8 warps][128] floats of shared memory.  Fixed order: xor-16 pair
// inside the warp, then warps 0..7 in sequence.
__device__ __forceinline__ float cta_sum_over_rows(const float part[8], float* red, int c) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float v[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) v[k] = part[k] + __shfl_xor_sync(0xffffffffu, part[k], 16);
  if (lane < 16) {
#pragma unroll
    for (int k = 0; k < 8; ++k) red[warp * kDim + c * 8 + k] = v[k];
  }
  __syncthreads();
  float s = 0.f;
  if (threadIdx.x < kDim) {
#pragma unroll
    for (int w = 0; w < 8; ++w) s += red[w * kDim + threadIdx.x];
  }
  __syncthreads();
  return s;
}

// kPerm: pool the permuted layout, reading Q through perm and writing the
// permuted rows to Qp.
template <bool kPerm>
__global__ void __launch_bounds__(kThreads) pool_q_kernel(const __nv_bfloat16* __restrict__ Q,
                                                          float* __restrict__ qpool, int N,
                                                          int nb, const int32_t* __restrict__ perm,
                                                          __nv_bfloat16* __restrict__ Qp) {
  __shared__ float red[8 * kDim];
  const int blk = blockIdx.x;
  const size_t bh = blockIdx.y;
  const int row0 = blk * kBlock;
  const int n = min(kBlock, N - row0);
  const int g = threadIdx.x >> 4, c = threadIdx.x & 15;
  uint4 rows[8];
  if constexpr (kPerm)
    load_block_rows_perm(Q + bh * N * kDim, perm + bh * N, row0, n, N, g, c, rows,
                         Qp + bh * N * kDim);
  else
    load_block_rows(Q + (bh * N + row0) * kDim, n, g, c, rows);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    float f[8];
    bf16x8_to_f32(rows[it], f);
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] += f[k];
  }
  const float s = cta_sum_over_rows(acc, red, c);
  if (threadIdx.x < kDim) qpool[(bh * nb + blk) * kDim + threadIdx.x] = s / static_cast<float>(n);
}

// 1024 threads: 8 groups of 128 dims; group gi sums blocks i = pb+gi, pb+gi+8, ...
__global__ void __launch_bounds__(1024) anchor_kernel(const float* __restrict__ qpool,
                                                      float* __restrict__ anchor, int N, int nb,
                                                      int pb) {
  __shared__ float part[8][kDim];
  const size_t bh = blockIdx.x;
  const int d = threadIdx.x & (kDim - 1), gi = threadIdx.x >> 7;
  const float* qp = qpool + bh * nb * kDim;
  float s = 0.f;
  for (int i = pb + gi; i < nb; i += 8) {
    const float n_i = static_cast<float>(min(kBlock, N - i * kBlock));
    s += __ldg(qp + static_cast<size_t>(i) * kDim + d) * n_i;
  }
  part[gi][d] = s;
  __syncthreads();
  if (gi == 0) {
    float t = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) t += part[k][d];
    anchor[bh * kDim + d] = t / static_cast<float>(N - pb * kBlock);
  }
}

// kVariant: 0 = anchor-weighted, 1 = mean-pooled; kPerm: the permuted layout
template <int kVariant, bool kPerm>
__global__ void __launch_bounds__(kThreads) summarize_kernel(
    const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V,
    const float* __restrict__ anchor, float* __restrict__ kpool, __nv_bfloat16* __restrict__ ksum,
    __nv_bfloat16* __restrict__ vsum, float* __restrict__ bias, float* __restrict__ kstat,
    float* __restrict__ vstat, float* __restrict__ lse_blk, int N, int nb, float scale,
    const int32_t* __restrict__ perm, __nv_bfloat16* __restrict__ Kp,
    __nv_bfloat16* __restrict__ Vp) {
  __shared__ float red[8 * kDim];
  __shared__ float xs[kBlock];
  __shared__ float stat[2];
  const int blk = blockIdx.x;
  const size_t bh = blockIdx.y;
  const int row0 = blk * kBlock;
  const int n = min(kBlock, N - row0);
  const int tid = threadIdx.x, g = tid >> 4, c = tid & 15;
  const int lane = tid & 31, warp = tid >> 5;

  uint4 kr[8], vr[8];
  if constexpr (kPerm) {   // K and V through perm, their copies to Kp, Vp
    load_block_rows_perm(K + bh * N * kDim, perm + bh * N, row0, n, N, g, c, kr,
                         Kp + bh * N * kDim);
    load_block_rows_perm(V + bh * N * kDim, perm + bh * N, row0, n, N, g, c, vr,
                         Vp + bh * N * kDim);
  } else {
    load_block_rows(K + (bh * N + row0) * kDim, n, g, c, kr);
    load_block_rows(V + (bh * N + row0) * kDim, n, g, c, vr);
  }

  float ks[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    float f[8];
    bf16x8_to_f32(kr[it], f);
#pragma unroll
    for (int k = 0; k < 8; ++k) ks[k] += f[k];
  }

  float kt[8], vt[8];
  float lse = 0.f;
  if (kVariant == 0) {
    float a[8];
    const float4* ap = reinterpret_cast<const float4*>(anchor + bh * kDim + c * 8);
    const float4 a0 = __ldg(ap), a1 = __ldg(ap + 1);
    a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
    a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
    // x_r = anchor . k_r * scale for the 8 rows of this thread's group
    float x[8];
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      float f[8];
      bf16x8_to_f32(kr[it], f);
      float p = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) p = fmaf(a[k], f[k], p);
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
      x[it] = p * scale;
    }
    if (c == 0) {
#pragma unroll
      for (int it = 0; it < 8; ++it) xs[g + 16 * it] = x[it];
    }
    __syncthreads();
    if (warp == 0) {  // block max and log-sum-exp over the n real rows
      float m = -INFINITY;
      for (int r = lane; r < n; r += 32) m = fmaxf(m, xs[r]);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float s = 0.f;
      for (int r = lane; r < n; r += 32) s += expf(xs[r] - m);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) stat[0] = m + logf(s);
    }
    __syncthreads();
    lse = stat[0];
#pragma unroll
    for (int k = 0; k < 8; ++k) { kt[k] = 0.f; vt[k] = 0.f; }
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int r = g + 16 * it;
      const float w = (r < n) ? expf(x[it] - lse) : 0.f;
      float fk[8], fv[8];
      bf16x8_to_f32(kr[it], fk);
      bf16x8_to_f32(vr[it], fv);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        kt[k] = fmaf(w, fk[k], kt[k]);
        vt[k] = fmaf(w, fv[k], vt[k]);
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) vt[k] = 0.f;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      float fv[8];
      bf16x8_to_f32(vr[it], fv);
#pragma unroll
      for (int k = 0; k < 8; ++k) vt[k] += fv[k];
    }
  }

  const float inv_n = 1.f / static_cast<float>(n);
  const float ksum_d = cta_sum_over_rows(ks, red, c);
  const float vt_d = cta_sum_over_rows(vt, red, c);
  float kt_d = 0.f;
  if (kVariant == 0) kt_d = cta_sum_over_rows(kt, red, c);

  const size_t o = (bh * nb + blk) * kDim + tid;
  if (tid < kDim) kpool[o] = ksum_d * inv_n;
  if (kVariant == 0) {
    // bias = LSE - anchor . bf16(k~) * scale  (bf16(k~) is what the MMA sees)
    const float kt_b = bf16_round(kt_d);
    float p = (tid < kDim) ? __ldg(anchor + bh * kDim + tid) * kt_b : 0.f;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
    if (lane == 0 && warp < 4) red[warp] = p;
    __syncthreads();
    if (tid < kDim) {
      ksum[o] = __float2bfloat16_rn(kt_d);
      vsum[o] = __float2bfloat16_rn(vt_d);
      if (kstat) {   // fp32 statistics for the summaries of partial blocks
        kstat[o] = kt_d;
        vstat[o] = vt_d;
      }
    }
    if (tid == 0) bias[bh * nb + blk] = lse - ((red[0] + red[1]) + (red[2] + red[3])) * scale;
    if (tid == 0 && lse_blk) lse_blk[bh * nb + blk] = lse;
  } else {
    if (tid < kDim) {
      ksum[o] = __float2bfloat16_rn(ksum_d * inv_n);
      vsum[o] = __float2bfloat16_rn(vt_d * inv_n);
      if (kstat) {
        kstat[o] = ksum_d * inv_n;
        vstat[o] = vt_d * inv_n;
      }
    }
    if (tid == 0) bias[bh * nb + blk] = logf(static_cast<float>(n));
    if (tid == 0 && lse_blk) lse_blk[bh * nb + blk] = logf(static_cast<float>(n));
  }
}

}  // namespace

cudaError_t launch_pool(const Shape& s, const void* Q, float* qpool, float* anchor,
                        cudaStream_t st, const int32_t* perm, void* Qp) {
  const dim3 grid(s.nb, s.B * s.H);
  if (perm)
    pool_q_kernel<true><<<grid, kThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(Q), qpool,
                                                   s.N, s.nb, perm,
                                                   static_cast<__nv_bfloat16*>(Qp));
  else
    pool_q_kernel<false><<<grid, kThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(Q), qpool,
                                                    s.N, s.nb, nullptr, nullptr);
  anchor_kernel<<<s.B * s.H, 1024, 0, st>>>(qpool, anchor, s.N, s.nb, s.pb);
  return cudaGetLastError();
}

cudaError_t launch_summarize(const Shape& s, const void* K, const void* V, const float* anchor,
                             float* kpool, void* ksum, void* vsum, float* bias, cudaStream_t st,
                             float* kstat, float* vstat, float* lse_blk, const int32_t* perm,
                             void* Kp_out, void* Vp_out) {
  const dim3 grid(s.nb, s.B * s.H);
  const float scale = 0.088388347648318440550f;  // 1 / sqrt(128)
  auto Kp = static_cast<const __nv_bfloat16*>(K);
  auto Vp = static_cast<const __nv_bfloat16*>(V);
  auto ks = static_cast<__nv_bfloat16*>(ksum);
  auto vs = static_cast<__nv_bfloat16*>(vsum);
  auto ko = static_cast<__nv_bfloat16*>(Kp_out);
  auto vo = static_cast<__nv_bfloat16*>(Vp_out);
  if (s.variant == 0 && perm)
    summarize_kernel<0, true><<<grid, kThreads, 0, st>>>(Kp, Vp, anchor, kpool, ks, vs, bias,
                                                         kstat, vstat, lse_blk, s.N, s.nb, scale,
                                                         perm, ko, vo);
  else if (s.variant == 0)
    summarize_kernel<0, false><<<grid, kThreads, 0, st>>>(Kp, Vp, anchor, kpool, ks, vs, bias,
                                                          kstat, vstat, lse_blk, s.N, s.nb, scale,
                                                          nullptr, nullptr, nullptr);
  else if (perm)
    summarize_kernel<1, true><<<grid, kThreads, 0, st>>>(Kp, Vp, anchor, kpool, ks, vs, bias,
                                                         kstat, vstat, lse_blk, s.N, s.nb, scale,
                                                         perm, ko, vo);
  else
    summarize_kernel<1, false><<<grid, kThreads, 0, st>>>(Kp, Vp, anchor, kpool, ks, vs, bias,
                                                          kstat, vstat, lse_blk, s.N, s.nb, scale,
                                                          nullptr, nullptr, nullptr);
  return cudaGetLastError();
}

}  // namespace bsa
