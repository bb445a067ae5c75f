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
// Rows of up to 3072 video key blocks take the scores from the tensor cores
// instead (select_tc_kernel, same phase 2):
//  * one CTA per (R query blocks, head), R = 32 or 16; the MMA puts 128 key
//    blocks on M (TMEM lanes) and the R query blocks on N, so the scores of
//    key chunk c sit in TMEM columns [c R, c R + R) and stay there until
//    every chunk is done;
//  * fp32-grade products from TF32 inputs: x = hi + lo with hi = x with its
//    low 13 mantissa bits cleared (a TF32 value exactly) and lo = x - hi
//    (exact in fp32; the tensor core keeps 11 significant bits of it, so it
//    is within 2^-20 |x|); q.k = hi_q.hi_k + hi_q.lo_k + lo_q.hi_k, the
//    dropped lo_q.lo_k being under 2^-20 |q_d k_d| as well;
//  * TMA brings fp32 tiles of 32 dimensions (one 128-byte swizzle row) x 128
//    pooled keys into a ring; four converter warps each take the rows of
//    their TMEM lane quarter, split them in registers and store hi and lo to
//    a TMEM tile (the MMA's A operand, so only the small query tile is read
//    from shared memory: with A in shared memory the 4 KB it reads per MMA
//    for only R columns bounded the score phase); one thread issues the MMAs;
//  * then per batch of 8 query blocks the 8 warps copy the batch's scores
//    from TMEM into shared memory (the staging space is free by then) and
//    each warp selects one row.
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

// Exclusive prefix sum of v over the lanes of the warp.
__device__ __forceinline__ int warp_excl_scan(int v, int lane) {
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x - v;
}

// Top-k of one row of nbv scores (in shared memory) by one warp.  Lane l keeps
// the keys of blocks l*kPerLane .. l*kPerLane + kPerLane - 1 in registers
// (nbv <= 32 * kPerLane), so lane-major order is ascending block order.
//  1. Bitwise binary search for the k_eff-th largest key T with warp-wide
//     counts over all keys while the range [T, T + 2^b) known to hold it
//     contains more than 64 keys (it narrows by one bit per pass; rows of
//     pooled scores get there in about ten passes).
//  2. The keys of that range go to the warp's 64-word buffer `cbuf`, two per
//     lane, and the search finishes on them (the keys above the range are
//     counted once).
//  3. Emission: every key above T, then the lowest-index keys equal to T,
//     each lane writing its own blocks at its exclusive prefix of the counts.
template <int kPerLane>
__device__ __forceinline__ void topk_row(const float* srow, int nbv, int k_eff, int pb,
                                         int32_t* row, int lane, uint32_t* cbuf) {
  static_assert(kPerLane <= 64, "64-bit lane masks");
  const int j0 = lane * kPerLane;
  uint32_t key[kPerLane];
#pragma unroll
  for (int e = 0; e < kPerLane; ++e)
    key[e] = (j0 + e < nbv) ? orderable_key(srow[j0 + e]) : 0u;   // 0 is below every real key
  uint32_t T = 0;
  int above = 0;       // keys at or above the top of the current range
  int at_least = nbv;  // keys >= T
  int b = 31;
  for (; b >= 0; --b) {
    const uint32_t cand = T | (1u << b);
    int c = 0;
#pragma unroll
    for (int e = 0; e < kPerLane; ++e) c += (key[e] >= cand) ? 1 : 0;
    c = __reduce_add_sync(0xffffffffu, c);
    if (c >= k_eff) {
      T = cand;
      at_least = c;
    } else {
      above = c;
    }
    if (at_least - above <= 64) break;
  }
  int gt, eq;
  if (b > 0) {
    // the range [T, T + 2^b) holds at most 64 keys: finish on those
    const uint32_t width = 1u << b;
    int own = 0;
#pragma unroll
    for (int e = 0; e < kPerLane; ++e) own += (j0 + e < nbv && key[e] - T < width) ? 1 : 0;
    int pos = warp_excl_scan(own, lane);
#pragma unroll
    for (int e = 0; e < kPerLane; ++e)
      if (j0 + e < nbv && key[e] - T < width) cbuf[pos++] = key[e];
    __syncwarp();
    const int nc = at_least - above;
    const uint32_t c0 = lane < nc ? cbuf[lane] : 0u;
    const uint32_t c1 = lane + 32 < nc ? cbuf[lane + 32] : 0u;
    __syncwarp();
    // every candidate lies below the keys counted in `above`
    for (--b; b >= 0; --b) {
      const uint32_t cand = T | (1u << b);
      const int c =
          above + __reduce_add_sync(0xffffffffu, (c0 >= cand ? 1 : 0) + (c1 >= cand ? 1 : 0));
      if (c >= k_eff) T = cand;
    }
    gt = above + __reduce_add_sync(0xffffffffu, (c0 > T ? 1 : 0) + (c1 > T ? 1 : 0));
    eq = __reduce_add_sync(0xffffffffu, (lane < nc && c0 == T ? 1 : 0) + (lane + 32 < nc && c1 == T ? 1 : 0));
  } else {
    int g = 0, q = 0;
#pragma unroll
    for (int e = 0; e < kPerLane; ++e) {
      g += (key[e] > T) ? 1 : 0;
      q += (j0 + e < nbv && key[e] == T) ? 1 : 0;
    }
    gt = __reduce_add_sync(0xffffffffu, g);
    eq = __reduce_add_sync(0xffffffffu, q);
  }
  (void)eq;
  const int need_eq = k_eff - gt;
  uint64_t gm = 0, em = 0;
#pragma unroll
  for (int e = 0; e < kPerLane; ++e) {
    gm |= static_cast<uint64_t>(key[e] > T) << e;
    em |= static_cast<uint64_t>(j0 + e < nbv && key[e] == T) << e;
  }
  // the lowest-index keys equal to T, as many as are needed
  const int ec = __popcll(em);
  int take = need_eq - warp_excl_scan(ec, lane);
  take = take < 0 ? 0 : (take > ec ? ec : take);
  uint64_t sel = gm;
  for (int t = 0; t < take; ++t) {
    const uint64_t low = em & (~em + 1);
    sel |= low;
    em ^= low;
  }
  int pos = pb + warp_excl_scan(__popcll(sel), lane);
  for (; sel; sel &= sel - 1) row[pos++] = pb + j0 + __ffsll(static_cast<long long>(sel)) - 1;
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

// One query block's selection from its scores in shared memory (both kernels).
template <int kPerLane, bool kThresh>
__device__ __forceinline__ void select_row(const float* srow, int i, size_t bh, int nb, int pb,
                                           int k_eff, int kcap, float tau, int32_t* idx,
                                           int32_t* cnt, int lane, uint32_t* cbuf) {
  const int nbv = nb - pb;
  int32_t* row = idx + (bh * nb + i) * kcap;
  if (i < pb) {  // dense-prefix query block: every block, no summaries
    for (int p = lane; p < kcap; p += 32) row[p] = (p < nb) ? p : -1;
    if (lane == 0) cnt[bh * nb + i] = nb;
    return;
  }
  int kept = k_eff;
  if constexpr (kThresh)
    kept = threshold_row(srow, nbv, tau, pb, row, lane);
  else if constexpr (kPerLane > 0)
    topk_row<kPerLane>(srow, nbv, k_eff, pb, row, lane, cbuf);
  else
    topk_row_smem(srow, nbv, k_eff, pb, row, lane);
  for (int p = lane; p < pb; p += 32) row[p] = p;
  for (int p = pb + kept + lane; p < kcap; p += 32) row[p] = -1;
  if (lane == 0) cnt[bh * nb + i] = pb + kept;
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
  float* sc = kc + kChunk * kPad;            // [R][nbv], then 64 words per warp
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
    select_row<kPerLane, kThresh>(sc + r * nbv, i, bh, nb, pb, k_eff, kcap, tau, idx, cnt, lane,
                                  reinterpret_cast<uint32_t*>(sc + R * nbv) + 64 * warp);
  }
}

// ---------------------------------------------------------- tensor-core scores

// warp 0 TMA, 1 MMA + TMEM, 4-7 convert; all select (8 warps with two CTAs
// per SM, 16 with one)
constexpr int kTcMaxWarps = 16;
constexpr uint32_t kKTile = 16384;  // 128 pooled keys x 32 fp32 (one swizzle row each)
constexpr int kTcMaxStages = 8;     // raw key tiles in flight
constexpr int kTcAStages = 2;       // converted key tiles (TMEM, 64 columns each)

struct TcCtl {
  uint64_t bfull, bconv, done;
  uint64_t full[kTcMaxStages], rempty[kTcMaxStages];
  uint64_t conv[kTcAStages], aempty[kTcAStages];
  uint32_t tmem_base;
  int abort_flag;
  uint32_t cbuf[kTcMaxWarps][64];   // per warp: the candidate keys of the top-k
};

struct TcCfg {
  int R;            // query blocks per CTA (MMA N)
  int warps;        // 8 (two CTAs per SM) or 16
  int stages;       // raw key tiles in flight
  uint32_t tcols;   // TMEM columns allocated (power of two)
  uint32_t acol;    // first TMEM column of the converted key tiles
  int sstride;      // floats per score row of a phase-2 batch
  uint32_t off_ring, off_ctl;
  size_t smem;
};

// Instruction descriptor, kind::tf32: D fp32, A/B TF32 (format code 2), both
// K-major, M and N given.  K is 8 per instruction.
__host__ __device__ constexpr uint32_t idesc_tf32_f32(uint32_t M, uint32_t N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::tf32.  A (M=128 rows x K=8) sits in
// TMEM with row i in lane i and one TF32 element per column (8 columns).
__device__ __forceinline__ void mma_tf32_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// In place: each float of the n4 float4s at `hi` becomes its TF32 head (low 13
// mantissa bits cleared); the remainder goes to the same place at `lo`.
__device__ __forceinline__ void split_tf32(uint8_t* hi, uint8_t* lo, int n4, int t, int nt) {
  float4* h4 = reinterpret_cast<float4*>(hi);
  float4* l4 = reinterpret_cast<float4*>(lo);
  for (int e = t; e < n4; e += nt) {
    const float4 x = h4[e];
    float4 h;
    h.x = __uint_as_float(__float_as_uint(x.x) & 0xffffe000u);
    h.y = __uint_as_float(__float_as_uint(x.y) & 0xffffe000u);
    h.z = __uint_as_float(__float_as_uint(x.z) & 0xffffe000u);
    h.w = __uint_as_float(__float_as_uint(x.w) & 0xffffe000u);
    h4[e] = h;
    l4[e] = make_float4(x.x - h.x, x.y - h.y, x.z - h.z, x.w - h.w);
  }
}

template <int kPerLane, bool kThresh, int kW>
__global__ void __launch_bounds__(kW * 32, kW == 8 ? 2 : 1)
    select_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k, int32_t* __restrict__ idx,
                     int32_t* __restrict__ cnt, int nb, int pb, int k_eff, int kcap,
                     const TcCfg cfg, float scale, float tau, int* dev_status) {
  extern __shared__ __align__(1024) uint8_t sm[];
  TcCtl* ctl = reinterpret_cast<TcCtl*>(sm + cfg.off_ctl);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y;
  const int R = cfg.R, S = cfg.stages;
  const int i0 = blockIdx.x * R;
  const int nbv = nb - pb;
  const int chunks = (nbv + kBlock - 1) / kBlock;
  const int T = chunks * 4;                       // key tiles: 4 per chunk of 128
  const uint32_t btile = static_cast<uint32_t>(R) * 128;   // one 32-dim slice of the query tile
  uint8_t* bhi = sm;
  uint8_t* blo = sm + 4 * btile;
  uint8_t* ring = sm + cfg.off_ring;

  if (tid == 0) {
    mbar_init(&ctl->bfull, 1);
    mbar_init(&ctl->bconv, 128);
    mbar_init(&ctl->done, 1);
    for (int st = 0; st < S; ++st) {
      mbar_init(&ctl->full[st], 1);
      mbar_init(&ctl->rempty[st], 128);
    }
    for (int st = 0; st < kTcAStages; ++st) {
      mbar_init(&ctl->conv[st], 128);
      mbar_init(&ctl->aempty[st], 1);
    }
    ctl->abort_flag = ((smem_u32(sm) & 1023u) != 0) ? 1 : 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, cfg.tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const WaitCtx wc{&ctl->abort_flag, dev_status};
  const bool run = ctl->abort_flag == 0;

  if (run && warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      mbar_arrive_expect_tx(&ctl->bfull, 4 * btile);
      for (int kb = 0; kb < 4; ++kb) tma_load_3d(bhi + kb * btile, &tm_q, &ctl->bfull, 32 * kb, i0, bh);
      int issued = 0;
      for (int it = 0; it < T; ++it) {
        const int st = it % S;
        if (it >= S && !mbar_wait(&ctl->rempty[st], ((it / S) - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(&ctl->full[st], kKTile);
        tma_load_3d(ring + st * kKTile, &tm_k, &ctl->full[st], 32 * (it & 3),
                    pb + kBlock * (it >> 2), bh);
        issued = it + 1;
      }
      // every issued load lands before the CTA moves on
      mbar_wait(&ctl->bfull, 0, wc);
      for (int k = (issued > S ? issued - S : 0); k < issued; ++k)
        mbar_wait(&ctl->full[k % S], (k / S) & 1, wc);
    }
  } else if (run && warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_tf32_f32(128, R);
      bool ok = mbar_wait(&ctl->bconv, 0, wc);
      for (int it = 0; it < T && ok; ++it) {
        const int sa = it % kTcAStages, kb = it & 3;
        if (!mbar_wait(&ctl->conv[sa], (it / kTcAStages) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + (it >> 2) * R;
        const uint32_t ahi = tmem + cfg.acol + 64 * sa, alo = ahi + 32;
        const uint32_t bh_ = smem_u32(bhi + kb * btile), bl_ = smem_u32(blo + kb * btile);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_tf32_ts(d, ahi + 8 * kk, smem_desc_sw128(bh_ + 32 * kk, 16, 1024), idesc,
                      (kb | kk) != 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_tf32_ts(d, ahi + 8 * kk, smem_desc_sw128(bl_ + 32 * kk, 16, 1024), idesc, 1u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_tf32_ts(d, alo + 8 * kk, smem_desc_sw128(bh_ + 32 * kk, 16, 1024), idesc, 1u);
        mma_commit(&ctl->aempty[sa]);
      }
      mma_commit(&ctl->done);
    }
  } else if (run && warp >= 4 && warp < 8) {
    const int t = tid - 128;
    bool ok = mbar_wait(&ctl->bfull, 0, wc);
    if (ok) split_tf32(bhi, blo, static_cast<int>(4 * btile / 16), t, 128);
    fence_proxy_async_smem();
    mbar_arrive(&ctl->bconv);
    // key row r of each tile (TMEM lane r): its 32 dimensions, split, to TMEM
    const int r = 32 * (warp & 3) + lane;
    const uint32_t lanes = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    for (int it = 0; it < T && ok; ++it) {
      const int st = it % S, sa = it % kTcAStages;
      if (!mbar_wait(&ctl->full[st], (it / S) & 1, wc)) { ok = false; break; }
      if (it >= kTcAStages && !mbar_wait(&ctl->aempty[sa], ((it / kTcAStages) - 1) & 1, wc)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint8_t* row = ring + st * kKTile + r * 128;
      uint32_t hi[32], lo[32];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float4 x = *reinterpret_cast<const float4*>(row + ((c ^ (r & 7)) << 4));
        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t h = __float_as_uint(xs[u]) & 0xffffe000u;
          hi[4 * c + u] = h;
          lo[4 * c + u] = __float_as_uint(xs[u] - __uint_as_float(h));
        }
      }
      mbar_arrive(&ctl->rempty[st]);   // the raw tile is in registers
      const uint32_t a = tmem + lanes + cfg.acol + 64 * sa;
      BSA_TMEM_ST_32(a, hi);
      BSA_TMEM_ST_32(a + 32, lo);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&ctl->conv[sa]);
    }
  }

  // ---------------------------------------------------------------- phase 2
  if (run) mbar_wait(&ctl->done, 0, wc);
  __syncthreads();
  tc_fence_after();
  if (ctl->abort_flag == 0) {
    float* sc = reinterpret_cast<float*>(sm);
    const int g = warp & 3, part = warp >> 2;
    for (int rb = 0; rb < R && i0 + rb < nb; rb += kW) {
      for (int c = part; c < chunks; c += kW / 4) {
        const int key = kBlock * c + 32 * g + lane;
#pragma unroll
        for (int r8 = 0; r8 < kW; r8 += 8) {
          uint32_t v[8];
          tmem_ld8(tmem + (static_cast<uint32_t>(32 * g) << 16) + c * R + rb + r8, v);
          tmem_wait_ld();
          if (key < nbv) {
#pragma unroll
            for (int r = 0; r < 8; ++r)
              sc[(r8 + r) * cfg.sstride + key] = __uint_as_float(v[r]) * scale;
          }
        }
      }
      __syncthreads();
      const int i = i0 + rb + warp;
      if (i < nb)
        select_row<kPerLane, kThresh>(sc + warp * cfg.sstride, i, bh, nb, pb, k_eff, kcap, tau,
                                      idx, cnt, lane, ctl->cbuf[warp]);
      __syncthreads();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, cfg.tcols);
}

// Tensor-core configuration for nbv video key blocks, or R = 0 when the
// scores and two converted key tiles do not fit in TMEM (more than 3072
// blocks).  `pair`: two CTAs per SM (each within 256 TMEM columns and half
// the shared memory), so one CTA's selection overlaps the other's score
// phase; otherwise one CTA per SM with all 512 columns and a deeper ring.  R
// query blocks per CTA share every key tile the CTA loads (32, else 16).
// The score batch of phase 2 (one row per warp) reuses the staging space.
TcCfg tc_config(int nbv, bool pair) {
  TcCfg c{};
  const int chunks = (nbv + kBlock - 1) / kBlock;
  const int cols = pair ? 256 : 512;
  const int acols = 64 * kTcAStages;
  if (nbv <= 0 || ((chunks * 16 + 63) & ~63) + acols > cols) return c;
  c.R = ((chunks * 32 + 63) & ~63) + acols <= cols ? 32 : 16;
  c.acol = static_cast<uint32_t>((chunks * c.R + 63) & ~63);
  const uint32_t need = c.acol + acols;
  c.tcols = 32;
  while (c.tcols < need) c.tcols <<= 1;
  c.sstride = (nbv + 3) & ~3;
  c.off_ring = static_cast<uint32_t>(c.R) * 1024;   // query tile: hi + lo, 4 slices each
  const size_t budget = pair ? 113 * 1024 : 224 * 1024;
  c.stages = kTcMaxStages;
  while (c.stages > 2 && c.off_ring + c.stages * kKTile + sizeof(TcCtl) > budget) --c.stages;
  c.off_ctl = c.off_ring + c.stages * kKTile;
  c.smem = c.off_ctl + sizeof(TcCtl);
  // one warp per row of a phase-2 batch: 16 where one CTA holds the SM and
  // a batch of 16 score rows fits, else 8
  const auto batch = [&](int w) { return static_cast<size_t>(w) * c.sstride * 4; };
  c.warps = (!pair && c.R % 16 == 0 && batch(16) <= c.off_ctl) ? 16 : 8;
  if (batch(c.warps) > c.off_ctl || c.smem > budget) c.R = 0;
  // one CTA per SM: ask for more than half of the SM's shared memory
  if (!pair && c.smem < 120 * 1024) c.smem = 120 * 1024;
  return c;
}

// Two CTAs per SM where they fit (measured at 56 heads: 75.7 against 118 us
// at 295 blocks per row, 648 against 674 us at 1045), else one.
TcCfg tc_config(int nbv) {
  const TcCfg p = tc_config(nbv, true);
  return p.R > 0 ? p : tc_config(nbv, false);
}

template <int kPerLane, bool kThresh, int kW>
cudaError_t launch_select_tc_w(const Shape& s, const SelectMaps& maps, const TcCfg& cfg,
                               int32_t* idx, int32_t* cnt, cudaStream_t st, float tau) {
  static std::atomic<bool> attr_set[64];
  cudaError_t e = once_per_device(attr_set, [] {
    return cudaFuncSetAttribute(select_tc_kernel<kPerLane, kThresh, kW>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, 225 * 1024);
  });
  if (e != cudaSuccess) return e;
  const dim3 grid((s.nb + cfg.R - 1) / cfg.R, s.B * s.H);
  const float scale = 0.088388347648318440550f;
  const int kcap = kThresh ? s.nb : s.kcap;
  select_tc_kernel<kPerLane, kThresh, kW><<<grid, kW * 32, cfg.smem, st>>>(
      maps.q, maps.k, idx, cnt, s.nb, s.pb, s.k_eff, kcap, cfg, scale, tau, s.dev_status);
  return cudaGetLastError();
}

template <int kPerLane, bool kThresh = false>
cudaError_t launch_select_tc(const Shape& s, const SelectMaps& maps, const TcCfg& cfg,
                             int32_t* idx, int32_t* cnt, cudaStream_t st, float tau = 0.f) {
  return cfg.warps == 16
             ? launch_select_tc_w<kPerLane, kThresh, 16>(s, maps, cfg, idx, cnt, st, tau)
             : launch_select_tc_w<kPerLane, kThresh, 8>(s, maps, cfg, idx, cnt, st, tau);
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
  const size_t fixed = static_cast<size_t>(kChunk) * kPad * 4 + kThreads / 32 * 64 * 4;
  int R = nbv < 512 ? 16 : 32;
  while (R > 1 && fixed + static_cast<size_t>(R) * (kPad + nbv) * 4 > 220 * 1024) --R;
  return R;
}

static size_t select_smem(int R, int nbv) {
  return (static_cast<size_t>(R) * kPad + kChunk * kPad + static_cast<size_t>(R) * nbv +
          kThreads / 32 * 64) *
         sizeof(float);
}

int select_tc_rows(const Shape& s) { return tc_config(s.nbv).R; }

cudaError_t launch_select_threshold(const Shape& s, float tau, const SelectMaps* maps,
                                    const float* qpool, const float* kpool, int32_t* idx,
                                    int32_t* cnt, cudaStream_t st) {
  const TcCfg cfg = tc_config(s.nbv);
  if (maps && cfg.R > 0) return launch_select_tc<0, true>(s, *maps, cfg, idx, cnt, st, tau);
  const int R = select_rows(s.nbv);
  return launch_select_t<0, true>(s, qpool, kpool, idx, cnt, R, select_smem(R, s.nbv), st, tau);
}

cudaError_t launch_select(const Shape& s, const SelectMaps* maps, const float* qpool,
                          const float* kpool, int32_t* idx, int32_t* cnt, cudaStream_t st) {
  const TcCfg cfg = tc_config(s.nbv);
  if (maps && cfg.R > 0) {
    // keys per lane: the smallest instantiation that holds the row (odd, so the
  // lanes' strided loads of their keys hit 32 different banks)
    if (s.nbv <= 32 * 9) return launch_select_tc<9>(s, *maps, cfg, idx, cnt, st);
    if (s.nbv <= 32 * 13) return launch_select_tc<13>(s, *maps, cfg, idx, cnt, st);
    if (s.nbv <= 32 * 17) return launch_select_tc<17>(s, *maps, cfg, idx, cnt, st);
    if (s.nbv <= 32 * 25) return launch_select_tc<25>(s, *maps, cfg, idx, cnt, st);
    if (s.nbv <= 32 * 35) return launch_select_tc<35>(s, *maps, cfg, idx, cnt, st);
    if (s.nbv <= 32 * 47) return launch_select_tc<47>(s, *maps, cfg, idx, cnt, st);
    return launch_select_tc<0>(s, *maps, cfg, idx, cnt, st);
  }
  const int R = select_rows(s.nbv);
  const size_t smem = select_smem(R, s.nbv);
  if (s.nbv <= 32 * 9) return launch_select_t<9>(s, qpool, kpool, idx, cnt, R, smem, st);
  if (s.nbv <= 32 * 13) return launch_select_t<13>(s, qpool, kpool, idx, cnt, R, smem, st);
  if (s.nbv <= 32 * 17) return launch_select_t<17>(s, qpool, kpool, idx, cnt, R, smem, st);
  if (s.nbv <= 32 * 25) return launch_select_t<25>(s, qpool, kpool, idx, cnt, R, smem, st);
  if (s.nbv <= 32 * 35) return launch_select_t<35>(s, qpool, kpool, idx, cnt, R, smem, st);
  if (s.nbv <= 32 * 47) return launch_select_t<47>(s, qpool, kpool, idx, cnt, R, smem, st);
  return launch_select_t<0>(s, qpool, kpool, idx, cnt, R, smem, st);
}

}  // namespace bsa
