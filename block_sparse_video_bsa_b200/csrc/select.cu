// Block score + per-query-block top-k ("each query block attends to its
// top-k key blocks", h3-sparse-attn 0.1.0, opening description).
//
// One CTA per (tile of R query blocks, head), 256 threads:
//  1. scores  S_ij = qpool_i . kpool_j / sqrt(128) in fp32 for every video
//     key block j >= pb, kept in shared memory (never written to HBM).  The
//     pooled keys stream through shared memory 128 blocks at a time
//     (coalesced 16-byte loads, rows padded against bank conflicts); each
//     thread forms the dot products of four query blocks with four key
//     blocks with packed fp32x2 FMAs (even and odd dimensions in two partial
//     sums, added at the end; a fixed order, so the result is deterministic).
//  2. one warp per query block finds the k_eff-th largest score as a 32-bit
//     order-preserving key by bitwise binary search (32 count passes,
//     __reduce_add_sync per pass, the row's keys held in registers), then
//     emits, in ascending j, every block above that key plus the
//     lowest-index blocks equal to it -- exactly "score descending, ties to
//     the lower index".
// Dense-prefix query blocks (i < pb) list every block.
//
// Threshold mode (content-adaptive count; "H3 Sparse Attention", WAS node
// page, "The inputs that matter": the kept share of key blocks is set by a
// threshold tau): phase 2 keeps, per query block, the video key blocks whose
// score is at least tau population standard deviations above the row's mean
// (all of them when the row's scores are all equal, the top-scoring one when
// none qualifies), so list lengths vary from row to row.
#include "bsa_device.cuh"
#include "bsa_kernels.h"

namespace bsa {

namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 128;              // key blocks per shared-memory chunk
constexpr int kPad = kDim + 4;           // padded row of 132 floats

// Top-k of one row of nbv scores (in shared memory) by warp `lane`s; the keys
// are copied to registers (kPerLane per lane, nbv <= 32 * kPerLane).
template <int kPerLane>
__device__ __forceinline__ void topk_row(const float* srow, int nbv, int k_eff, int pb,
                                         int32_t* row, int lane) {
  uint32_t key[kPerLane];
#pragma unroll
  for (int e = 0; e < kPerLane; ++e) {
    const int j = lane + 32 * e;
    key[e] = (j < nbv) ? orderable_key(srow[j]) : 0u;   // 0 is below every real key
  }
  // k_eff-th largest key T: largest T with #{key >= T} >= k_eff.
  uint32_t T = 0;
  for (int b = 31; b >= 0; --b) {
    const uint32_t cand = T | (1u << b);
    int c = 0;
#pragma unroll
    for (int e = 0; e < kPerLane; ++e) c += (key[e] >= cand) ? 1 : 0;
    c = __reduce_add_sync(0xffffffffu, c);
    if (c >= k_eff) T = cand;
  }
  int gt = 0;
#pragma unroll
  for (int e = 0; e < kPerLane; ++e) gt += (key[e] > T) ? 1 : 0;
  gt = __reduce_add_sync(0xffffffffu, gt);
  const int need_eq = k_eff - gt;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int out = 0, eq_seen = 0;
#pragma unroll
  for (int e = 0; e < kPerLane; ++e) {
    if (32 * e >= nbv) break;
    const int j = lane + 32 * e;
    const bool valid = j < nbv;
    const bool is_gt = valid && key[e] > T;
    const bool is_eq = valid && key[e] == T;
    const uint32_t eqm = __ballot_sync(0xffffffffu, is_eq);
    const bool sel = is_gt || (is_eq && (eq_seen + __popc(eqm & lt_mask)) < need_eq);
    const uint32_t selm = __ballot_sync(0xffffffffu, sel);
    if (sel) row[pb + out + __popc(selm & lt_mask)] = pb + j;
    out += __popc(selm);
    eq_seen += __popc(eqm);
  }
}

// Same selection for rows too long to keep in registers (keys re-read from
// shared memory on every pass).
__device__ __forceinline__ void topk_row_smem(const float* srow, int nbv, int k_eff, int pb,
                                              int32_t* row, int lane) {
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
}

// Threshold selection of one row of nbv scores (in shared memory) by one
// warp.  The sums are xor-butterfly reductions, so every lane holds the same
// bits of the mean and deviation and takes the same decisions.  Writes the
// kept blocks in ascending order at row[pb...] and returns how many.
__device__ __forceinline__ int threshold_row(const float* srow, int nbv, float tau, int pb,
                                             int32_t* row, int lane) {
  float sum = 0.f, mx = -INFINITY, mn = INFINITY;
  for (int j = lane; j < nbv; j += 32) {
    const float x = srow[j];
    sum += x;
    mx = fmaxf(mx, x);
    mn = fminf(mn, x);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  const float mean = sum / static_cast<float>(nbv);
  float ss = 0.f;
  for (int j = lane; j < nbv; j += 32) {
    const float dev = srow[j] - mean;
    ss = fmaf(dev, dev, ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float margin = tau * sqrtf(ss / static_cast<float>(nbv));
  const bool all = (mx == mn);           // no contrast: every block
  const uint32_t lt_mask = (1u << lane) - 1u;
  int out = 0;
  for (int base = 0; base < nbv; base += 32) {
    const int j = base + lane;
    const bool sel = j < nbv && (all || srow[j] - mean >= margin);
    const uint32_t selm = __ballot_sync(0xffffffffu, sel);
    if (sel) row[pb + out + __popc(selm & lt_mask)] = pb + j;
    out += __popc(selm);
  }
  if (out == 0) {
    // floor: the first block whose score equals the row maximum
    int first = nbv;
    for (int base = 0; base < nbv && first == nbv; base += 32) {
      const int j = base + lane;
      const uint32_t m = __ballot_sync(0xffffffffu, j < nbv && srow[j] == mx);
      if (m) first = base + __ffs(m) - 1;
    }
    if (lane == 0) row[pb] = pb + min(first, nbv - 1);
    out = 1;
  }
  return out;
}

// kPerLane: keys per lane of the top-k search (0 = keys stay in shared
// memory); kThresh: threshold mode (tau used, k_eff unused, kcap = nb).
template <int kPerLane, bool kThresh>
__global__ void __launch_bounds__(kThreads) select_kernel(const float* __restrict__ qpool,
                                                          const float* __restrict__ kpool,
                                                          int32_t* __restrict__ idx,
                                                          int32_t* __restrict__ cnt, int nb, int pb,
                                                          int k_eff, int kcap, int R, float scale,
                                                          float tau) {
  extern __shared__ float smem[];
  const int nbv = nb - pb;
  float* qp = smem;                          // [R][kPad]
  float* kc = qp + R * kPad;                 // [kChunk][kPad]
  float* sc = kc + kChunk * kPad;            // [R][nbv]
  const size_t bh = blockIdx.y;
  const int i0 = blockIdx.x * R;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  bool any_video = false;
  for (int r = 0; r < R; ++r) any_video |= (i0 + r >= pb && i0 + r < nb);

  if (any_video) {
    for (int e = tid; e < R * (kDim / 4); e += kThreads) {
      const int r = e / (kDim / 4), d4 = e % (kDim / 4);
      const int i = min(i0 + r, nb - 1);
      *reinterpret_cast<float4*>(qp + r * kPad + 4 * d4) =
          __ldg(reinterpret_cast<const float4*>(qpool + (bh * nb + i) * kDim) + d4);
    }
    // thread -> 4 query blocks (rows 4*warp .. 4*warp+3) x 4 key blocks of the
    // chunk (lane, lane+32, lane+64, lane+96): 16 dot products per thread, so
    // each 16-byte shared load feeds four of them.  Every dot product keeps
    // even and odd dimensions in two partial sums added at the end (a fixed
    // order: the result is deterministic).
    const int rg = warp;   // row group
    for (int c0 = 0; c0 < nbv; c0 += kChunk) {
      __syncthreads();   // previous chunk fully used (and qp written, first time)
      const int rows = min(kChunk, nbv - c0);
      for (int e = tid; e < rows * (kDim / 4); e += kThreads) {
        const int r = e / (kDim / 4), d4 = e % (kDim / 4);
        *reinterpret_cast<float4*>(kc + r * kPad + 4 * d4) = __ldg(
            reinterpret_cast<const float4*>(kpool + (bh * nb + pb + c0 + r) * kDim) + d4);
      }
      __syncthreads();
      if (4 * rg < R) {
        float2 acc[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) acc[a][b] = make_float2(0.f, 0.f);
        const float* q0 = qp + (4 * rg) * kPad;
#pragma unroll 4
        for (int d4 = 0; d4 < kDim / 4; ++d4) {
          float4 x[4], k[4];
#pragma unroll
          for (int a = 0; a < 4; ++a) x[a] = *reinterpret_cast<const float4*>(q0 + a * kPad + 4 * d4);
#pragma unroll
          for (int b = 0; b < 4; ++b)
            k[b] = *reinterpret_cast<const float4*>(kc + (lane + 32 * b) * kPad + 4 * d4);
#pragma unroll
          for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              acc[a][b] = fma2(make_float2(x[a].x, x[a].y), make_float2(k[b].x, k[b].y), acc[a][b]);
              acc[a][b] = fma2(make_float2(x[a].z, x[a].w), make_float2(k[b].z, k[b].w), acc[a][b]);
            }
        }
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          const int r = 4 * rg + a;
          if (r >= R) break;
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int kk = lane + 32 * b;
            if (kk < rows) sc[r * nbv + c0 + kk] = (acc[a][b].x + acc[a][b].y) * scale;
          }
        }
      }
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
    int kept = k_eff;
    if constexpr (kThresh)
      kept = threshold_row(sc + r * nbv, nbv, tau, pb, row, lane);
    else if constexpr (kPerLane > 0)
      topk_row<kPerLane>(sc + r * nbv, nbv, k_eff, pb, row, lane);
    else
      topk_row_smem(sc + r * nbv, nbv, k_eff, pb, row, lane);
    for (int p = lane; p < pb; p += 32) row[p] = p;
    for (int p = pb + kept + lane; p < kcap; p += 32) row[p] = -1;
    if (lane == 0) cnt[bh * nb + i] = pb + kept;
  }
}

template <int kPerLane, bool kThresh = false>
cudaError_t launch_select_t(const Shape& s, const float* qpool, const float* kpool, int32_t* idx,
                            int32_t* cnt, int R, size_t smem, cudaStream_t st, float tau = 0.f) {
  static std::atomic<bool> attr_set[64];
  cudaError_t e = once_per_device(attr_set, [] {
    return cudaFuncSetAttribute(select_kernel<kPerLane, kThresh>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024);
  });
  if (e != cudaSuccess) return e;
  const dim3 grid((s.nb + R - 1) / R, s.B * s.H);
  const float scale = 0.088388347648318440550f;
  const int kcap = kThresh ? s.nb : s.kcap;
  select_kernel<kPerLane, kThresh><<<grid, kThreads, smem, st>>>(qpool, kpool, idx, cnt, s.nb,
                                                                 s.pb, s.k_eff, kcap, R, scale,
                                                                 tau);
  return cudaGetLastError();
}

}  // namespace

// Query blocks per CTA: 16 for rows of fewer than 512 blocks (two CTAs fit
// on an SM), else 32 (four per warp in the score phase: each chunk of pooled
// keys serves twice the rows); fewer when a row of scores is long, so the
// tile stays within the shared memory of one CTA (at least one row: N <=
// 2^21 keeps a row under 64 KB).  Measured at 56 heads: 0.113 against 0.149
// ms with 16 and 32 rows at 295 blocks, 1.29 against 1.13 ms at 1045.
static int select_rows(int nbv) {
  const size_t fixed = static_cast<size_t>(kChunk) * kPad * 4;
  int R = nbv < 512 ? 16 : 32;
  while (R > 1 && fixed + static_cast<size_t>(R) * (kPad + nbv) * 4 > 220 * 1024) --R;
  return R;
}

static size_t select_smem(int R, int nbv) {
  return (static_cast<size_t>(R) * kPad + kChunk * kPad + static_cast<size_t>(R) * nbv) *
         sizeof(float);
}

cudaError_t launch_select_threshold(const Shape& s, float tau, const float* qpool,
                                    const float* kpool, int32_t* idx, int32_t* cnt,
                                    cudaStream_t st) {
  const int R = select_rows(s.nbv);
  return launch_select_t<0, true>(s, qpool, kpool, idx, cnt, R, select_smem(R, s.nbv), st, tau);
}

cudaError_t launch_select(const Shape& s, const float* qpool, const float* kpool, int32_t* idx,
                          int32_t* cnt, cudaStream_t st) {
  const int R = select_rows(s.nbv);
  const size_t smem = select_smem(R, s.nbv);
  // keys per lane: the smallest instantiation that holds the row
  if (s.nbv <= 32 * 8) return launch_select_t<8>(s, qpool, kpool, idx, cnt, R, smem, st);
  if (s.nbv <= 32 * 12) return launch_select_t<12>(s, qpool, kpool, idx, cnt, R, smem, st);
  if (s.nbv <= 32 * 16) return launch_select_t<16>(s, qpool, kpool, idx, cnt, R, smem, st);
  if (s.nbv <= 32 * 24) return launch_select_t<24>(s, qpool, kpool, idx, cnt, R, smem, st);
  if (s.nbv <= 32 * 34) return launch_select_t<34>(s, qpool, kpool, idx, cnt, R, smem, st);
  if (s.nbv <= 32 * 48) return launch_select_t<48>(s, qpool, kpool, idx, cnt, R, smem, st);
  return launch_select_t<0>(s, qpool, kpool, idx, cnt, R, smem, st);
}

}  // namespace bsa
