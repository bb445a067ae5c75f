// Block score + per-query-block top-k ("each query block attends to its
// top-k key blocks", h3-sparse-attn 0.1.0, opening description).
//
// One CTA per (tile of R query blocks, head), 256 threads:
//  1. scores  S_ij = qpool_i . kpool_j / sqrt(128) in fp32 for every video
//     key block j >= pb, kept in shared memory (never written to HBM);
//     128-term dot products summed in a fixed order (deterministic).
//  2. one warp per query block finds the k_eff-th largest score as a 32-bit
//     order-preserving key by bitwise binary search (32 count passes,
//     __reduce_add_sync per pass), then emits, in ascending j, every block
//     above that key plus the lowest-index blocks equal to it -- exactly
//     "score descending, ties to the lower index".
// Dense-prefix query blocks (i < pb) list every block.
#include "bsa_device.cuh"
#include "bsa_kernels.h"

namespace bsa {

namespace {

constexpr int kThreads = 256;
constexpr int kMaxRows = 8;

__global__ void __launch_bounds__(kThreads) select_kernel(const float* __restrict__ qpool,
                                                          const float* __restrict__ kpool,
                                                          int32_t* __restrict__ idx,
                                                          int32_t* __restrict__ cnt, int nb, int pb,
                                                          int k_eff, int kcap, int R, float scale) {
  extern __shared__ float smem[];
  float* qp = smem;                 // [R][128]
  float* sc = smem + R * kDim;      // [R][nbv]
  const int nbv = nb - pb;
  const size_t bh = blockIdx.y;
  const int i0 = blockIdx.x * R;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  bool any_video = false;
  for (int r = 0; r < R; ++r) any_video |= (i0 + r >= pb && i0 + r < nb);

  if (any_video) {
    for (int e = tid; e < R * kDim; e += kThreads) {
      const int r = e / kDim, d = e % kDim;
      const int i = min(i0 + r, nb - 1);
      qp[e] = __ldg(qpool + (bh * nb + i) * kDim + d);
    }
    __syncthreads();
    for (int jj = tid; jj < nbv; jj += kThreads) {
      const float4* kp = reinterpret_cast<const float4*>(kpool + (bh * nb + pb + jj) * kDim);
      float acc[kMaxRows];
#pragma unroll
      for (int r = 0; r < kMaxRows; ++r) acc[r] = 0.f;
#pragma unroll 4
      for (int d4 = 0; d4 < kDim / 4; ++d4) {
        const float4 k4 = __ldg(kp + d4);
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r) {
          if (r < R) {
            const float4 q4 = *reinterpret_cast<const float4*>(qp + r * kDim + d4 * 4);
            acc[r] = fmaf(q4.x, k4.x, acc[r]);
            acc[r] = fmaf(q4.y, k4.y, acc[r]);
            acc[r] = fmaf(q4.z, k4.z, acc[r]);
            acc[r] = fmaf(q4.w, k4.w, acc[r]);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < kMaxRows; ++r)
        if (r < R) sc[r * nbv + jj] = acc[r] * scale;
    }
    __syncthreads();
  }

  // One warp per query block of the tile.
  for (int r = warp; r < R; r += kThreads / 32) {
    const int i = i0 + r;
    if (i >= nb) break;
    int32_t* row = idx + (bh * nb + i) * kcap;
    if (i < pb) {  // dense-prefix query block: every block, no summaries
      for (int p = lane; p < kcap; p += 32) row[p] = (p < nb) ? p : -1;
      if (lane == 0) cnt[bh * nb + i] = nb;
      continue;
    }
    const float* srow = sc + r * nbv;
    // k_eff-th largest key T: largest T with #{key >= T} >= k_eff.
    uint32_t T = 0;
    for (int b = 31; b >= 0; --b) {
      const uint32_t cand = T | (1u << b);
      int c = 0;
      for (int j = lane; j < nbv; j += 32) c += (orderable_key(srow[j]) >= cand) ? 1 : 0;
      c = __reduce_add_sync(0xffffffffu, c);
      if (c >= k_eff) T = cand;
    }
    int gt = 0;
    for (int j = lane; j < nbv; j += 32) gt += (orderable_key(srow[j]) > T) ? 1 : 0;
    gt = __reduce_add_sync(0xffffffffu, gt);
    const int need_eq = k_eff - gt;
    const uint32_t lt_mask = (1u << lane) - 1u;
    int out = 0, eq_seen = 0;
    for (int base = 0; base < nbv; base += 32) {
      const int j = base + lane;
      const uint32_t u = (j < nbv) ? orderable_key(srow[j]) : 0u;
      const bool is_gt = (j < nbv) && (u > T);
      const bool is_eq = (j < nbv) && (u == T);
      const uint32_t eqm = __ballot_sync(0xffffffffu, is_eq);
      const bool sel = is_gt || (is_eq && (eq_seen + __popc(eqm & lt_mask)) < need_eq);
      const uint32_t selm = __ballot_sync(0xffffffffu, sel);
      if (sel) row[pb + out + __popc(selm & lt_mask)] = pb + j;
      out += __popc(selm);
      eq_seen += __popc(eqm);
    }
    for (int p = lane; p < pb; p += 32) row[p] = p;
    for (int p = pb + k_eff + lane; p < kcap; p += 32) row[p] = -1;
    if (lane == 0) cnt[bh * nb + i] = pb + k_eff;
  }
}

}  // namespace

// Rows per CTA: up to 8, fewer when a row of scores is large, so the score
// tile stays within 160 KB of shared memory.
static int select_rows(int nbv) {
  const int by_smem = (160 * 1024) / (nbv * 4 + kDim * 4);
  return by_smem < 1 ? 1 : (by_smem > kMaxRows ? kMaxRows : by_smem);
}

cudaError_t launch_select(const Shape& s, const float* qpool, const float* kpool, int32_t* idx,
                          int32_t* cnt, cudaStream_t st) {
  const int R = select_rows(s.nbv);
  const size_t smem = static_cast<size_t>(R) * (kDim + s.nbv) * sizeof(float);
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         200 * 1024);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const dim3 grid((s.nb + R - 1) / R, s.B * s.H);
  const float scale = 0.088388347648318440550f;
  select_kernel<<<grid, kThreads, smem, st>>>(qpool, kpool, idx, cnt, s.nb, s.pb, s.k_eff, s.kcap,
                                              R, scale);
  return cudaGetLastError();
}

}  // namespace bsa
