// Extra top-scoring tokens per query block, and the summary rows of the
// blocks that lose tokens to them.
//
// "H3 Sparse Attention" (comfy.icu, WAS node page), section "The inputs that
// matter": besides its chosen blocks, each query block reads a number of
// individually chosen top-scoring tokens (`extra_tokens`).  This library's
// readings: token u scores s_iu = qhat_i . k_u / sqrt(d); the candidates are
// the video tokens of the blocks not listed for query block i; the n_extra
// highest scores are taken, ties to the lower token index; an extra token is
// read exactly, so the summary row of its block stands for the block's
// remaining tokens only (the same summary definition over fewer tokens, and no
// row once every token of the block is extra).
//
//  select_extra_kernel   one CTA per (head, 128 video query blocks).  Token
//                        scores on tcgen05: A = qhat of the 128 query blocks
//                        split into bf16 hi + lo (qhat ~= hi + lo to ~16 bits;
//                        K is exact bf16), B = one 128-token key block from
//                        a 4-stage TMA ring, D = 128 x 128 fp32 in TMEM
//                        (double buffered).  One thread per query block keeps
//                        a running threshold and appends the candidates above
//                        it to its own buffer in global memory as 64-bit keys
//                        (order-preserving score bits << 32 | ~token, so a
//                        larger key is a higher score, then a lower index);
//                        when a buffer fills, the warp compacts it to the
//                        n_extra largest keys by an 8-bit radix select and
//                        raises the threshold to the smallest kept key.  The
//                        kept tokens are written in ascending order.
//  extra_summary_kernel  one CTA per video query block: the extra tokens form
//                        runs by block (the list is ascending); for each
//                        block that keeps some tokens, its summary over the
//                        remaining tokens is a downdate of the full block's
//                        fp32 statistics by the extra tokens (anchor variant:
//                        weights exp(x_u - LSE_j) of the extra tokens removed
//                        from the softmax-weighted sums; mean variant: the
//                        extra tokens removed from the sums), recomputed from
//                        the remaining rows when the remaining share of the
//                        block's anchor mass is under 2^-6 (where the
//                        subtraction would lose precision).
#include "bsa_device.cuh"
#include "bsa_kernels.h"

namespace bsa {

namespace {

constexpr int kSelThreads = 192;   // warps 0-3 select, 4 producer, 5 MMA
constexpr int kSelProducerWarp = 4;
constexpr int kSelMmaWarp = 5;
constexpr int kSelRing = 4;
constexpr uint32_t kTileB = 32768;   // 128 x 128 bf16
constexpr uint32_t kHalfB = 16384;   // 128 rows x 64 bf16 (one 128-byte swizzle atom wide)
constexpr uint32_t kOffAhi = 0;
constexpr uint32_t kOffAlo = kTileB;
constexpr uint32_t kOffRingB = 2 * kTileB;
constexpr uint32_t kOffSelCtl = kOffRingB + kSelRing * kTileB;
constexpr uint32_t kSelTmemCols = 256;

struct SelCtl {
  uint64_t full[kSelRing], empty[kSelRing];
  uint64_t d_full[2], d_empty[2];
  uint64_t fin;
  uint32_t tmem_base;
  int abort_flag;
  int skip;
  uint32_t scratch[4][512];   // per selection warp: radix histogram / sort buffer
};
static_assert(kOffSelCtl + sizeof(SelCtl) <= 227 * 1024, "shared memory budget");

struct SelArgs {
  const float* qpool;          // [BH, nb, 128]
  const int32_t* idx;          // [BH, nb, kcap]
  const int32_t* cnt;          // [BH, nb]
  unsigned long long* cand;    // [BH * nbv, kCap] candidate buffers
  int32_t* extra;              // [BH, nb, n_extra]
  int32_t* ecnt;               // [BH, nb]
  int* dev_status;
  int N, nb, pb, nbv, kcap, n_extra;
};

// 16-byte chunk c16 (0..15) of row r of a 128 x 128 bf16 tile in the 128-byte
// swizzled K-major layout the TMA writes (two 64-column boxes of 16 KB).
__device__ __forceinline__ uint32_t swz128(int r, int c16) {
  return static_cast<uint32_t>((c16 >> 3) * kHalfB + r * 128 + (((c16 & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ bool sel_wait(uint64_t* bar, uint32_t parity, const WaitCtx& wc) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc));
}

// Inverse of orderable_key on the score half of a candidate key.
__device__ __forceinline__ float key_score(unsigned long long key) {
  const uint32_t k = static_cast<uint32_t>(key >> 32);
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Warp-cooperative: the `target` largest of the `count` keys in buf[0..count)
// (all distinct, non-zero), left in buf[0..target) in any order.  Returns the
// smallest kept key.  8-bit radix select over the 64-bit keys, histograms in
// the warp's shared scratch.  Requires target <= count <= 32 * kSlots.
template <int kSlots>
__device__ unsigned long long compact_keys(unsigned long long* buf, int count, int target,
                                           uint32_t* hist) {
  const int lane = threadIdx.x & 31;
  __syncwarp();   // the owner's appends are visible to every lane
  unsigned long long e[kSlots];
#pragma unroll
  for (int k = 0; k < kSlots; ++k) {
    const int p = lane + 32 * k;
    e[k] = p < count ? buf[p] : 0ull;
  }
  __syncwarp();
  unsigned long long prefix = 0, pmask = 0;
  int krem = target;
#pragma unroll 1
  for (int shift = 56; shift >= 0; shift -= 8) {
#pragma unroll
    for (int b = 0; b < 8; ++b) hist[lane * 8 + b] = 0;
    __syncwarp();
#pragma unroll
    for (int k = 0; k < kSlots; ++k)
      if (e[k] != 0ull && (e[k] & pmask) == prefix)
        atomicAdd(&hist[static_cast<uint32_t>(e[k] >> shift) & 255u], 1u);
    __syncwarp();
    // lane l scans bins 255 - 8l down to 248 - 8l (descending digits)
    uint32_t h[8], run = 0;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      h[b] = hist[255 - (lane * 8 + b)];
      run += h[b];
    }
    uint32_t incl = run;   // inclusive scan over lanes (higher digits first)
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const uint32_t excl = incl - run;
    // the lane whose range holds the krem-th key (counting from the top)
    const bool mine = excl < static_cast<uint32_t>(krem) && static_cast<uint32_t>(krem) <= incl;
    const uint32_t owner = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    uint32_t digit = 0, above = 0;
    if (lane == owner) {
      uint32_t acc = excl;
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        if (acc + h[b] >= static_cast<uint32_t>(krem)) {
          digit = 255 - (lane * 8 + b);
          above = acc;
          break;
        }
        acc += h[b];
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, owner);
    above = __shfl_sync(0xffffffffu, above, owner);
    krem -= static_cast<int>(above);
    prefix |= static_cast<unsigned long long>(digit) << shift;
    pmask |= 0xffull << shift;
    __syncwarp();
  }
  // prefix is now the exact target-th largest key: keep e >= prefix
  int out = 0;
#pragma unroll
  for (int k = 0; k < kSlots; ++k) {
    const bool keep = e[k] != 0ull && e[k] >= prefix;
    const uint32_t m = __ballot_sync(0xffffffffu, keep);
    if (keep) buf[out + __popc(m & ((1u << lane) - 1u))] = e[k];
    out += __popc(m);
  }
  __syncwarp();
  return prefix;
}

template <int kCap>
__global__ void __launch_bounds__(kSelThreads, 1)
    select_extra_kernel(const __grid_constant__ CUtensorMap tm_k, const SelArgs a) {
  extern __shared__ __align__(1024) uint8_t sm[];
  SelCtl* ctl = reinterpret_cast<SelCtl*>(sm + kOffSelCtl);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y;
  const int i0 = a.pb + blockIdx.x * kBlock;          // first query block of the tile
  const int rows = min(kBlock, a.nb - i0);

  if (tid == 0) {
    const bool bad_align = (smem_u32(sm) & 1023u) != 0;
    if (bad_align && a.dev_status) atomicExch(a.dev_status, kErrTimeout);
    ctl->skip = (bad_align || (a.dev_status && *reinterpret_cast<volatile int*>(a.dev_status) != 0))
                    ? 1 : 0;
  }
  // dense-prefix query blocks take no extra tokens
  if (blockIdx.x == 0) {
    for (int e = tid; e < a.pb * a.n_extra; e += kSelThreads)
      a.extra[(static_cast<size_t>(bh) * a.nb) * a.n_extra + e] = -1;
    for (int i = tid; i < a.pb; i += kSelThreads) a.ecnt[static_cast<size_t>(bh) * a.nb + i] = 0;
  }
  __syncthreads();
  if (ctl->skip) return;

  // A operands: qhat of the tile's query blocks as bf16 hi and lo parts.
  for (int e = tid; e < kBlock * 16; e += kSelThreads) {
    const int r = e >> 4, c16 = e & 15;
    float q[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (r < rows) {
      const float4* src = reinterpret_cast<const float4*>(
          a.qpool + (static_cast<size_t>(bh) * a.nb + i0 + r) * kDim + c16 * 8);
      const float4 x0 = __ldg(src), x1 = __ldg(src + 1);
      q[0] = x0.x; q[1] = x0.y; q[2] = x0.z; q[3] = x0.w;
      q[4] = x1.x; q[5] = x1.y; q[6] = x1.z; q[7] = x1.w;
    }
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float h0 = bf16_round(q[2 * k]), h1 = bf16_round(q[2 * k + 1]);
      hi[k] = pack_bf16x2(h0, h1);
      lo[k] = pack_bf16x2(q[2 * k] - h0, q[2 * k + 1] - h1);
    }
    *reinterpret_cast<uint4*>(sm + kOffAhi + swz128(r, c16)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(sm + kOffAlo + swz128(r, c16)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
  fence_proxy_async_smem();
  if (tid == 0) {
    for (int s = 0; s < kSelRing; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->d_full[b], 1);
      mbar_init(&ctl->d_empty[b], kBlock);
    }
    mbar_init(&ctl->fin, 1);
    ctl->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kSelMmaWarp) {
    tmem_alloc(&ctl->tmem_base, kSelTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const WaitCtx wc{&ctl->abort_flag, a.dev_status};
  const int nblk = a.nbv;   // key blocks pb .. nb-1

  if (warp == kSelProducerWarp) {
    if (lane == 0) {
      prefetch_tensormap(&tm_k);
      bool ok = true;
      for (int it = 0; it < nblk && ok; ++it) {
        const int stage = it % kSelRing;
        if (it >= kSelRing && !mbar_wait(&ctl->empty[stage], ((it / kSelRing) - 1) & 1, wc)) {
          ok = false;
          break;
        }
        uint8_t* dst = sm + kOffRingB + stage * kTileB;
        const int row = (a.pb + it) * kBlock;
        mbar_arrive_expect_tx(&ctl->full[stage], kTileB);
        tma_load_3d(dst, &tm_k, &ctl->full[stage], 0, row, bh);
        tma_load_3d(dst + kHalfB, &tm_k, &ctl->full[stage], 64, row, bh);
      }
      // every issued load lands before the CTA exits
      const int issued = nblk;
      for (int k = (issued > kSelRing ? issued - kSelRing : 0); k < issued; ++k)
        mbar_wait(&ctl->full[k % kSelRing], (k / kSelRing) & 1, wc);
    }
  } else if (warp == kSelMmaWarp) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 128, 0);
      const uint32_t ahi = smem_u32(sm + kOffAhi), alo = smem_u32(sm + kOffAlo);
      bool ok = true;
      for (int it = 0; it < nblk && ok; ++it) {
        const int stage = it % kSelRing, b = it & 1;
        if (!mbar_wait(&ctl->full[stage], (it / kSelRing) & 1, wc)) { ok = false; break; }
        if (it >= 2 && !mbar_wait(&ctl->d_empty[b], ((it >> 1) - 1) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kaddr = smem_u32(sm + kOffRingB + stage * kTileB);
        const uint32_t d = tmem + b * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfB + (kk & 3) * 32;
          mma_bf16_ss(d, smem_desc_sw128(ahi + off, 16, 1024), smem_desc_sw128(kaddr + off, 16, 1024),
                      idesc, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfB + (kk & 3) * 32;
          mma_bf16_ss(d, smem_desc_sw128(alo + off, 16, 1024), smem_desc_sw128(kaddr + off, 16, 1024),
                      idesc, 1u);
        }
        mma_commit(&ctl->d_full[b]);
        mma_commit(&ctl->empty[stage]);
      }
      mma_commit(&ctl->fin);
      mbar_wait(&ctl->fin, 0, wc);
    }
  } else {
    // ------------------------------------------------------------ selection
    constexpr int kSlots = kCap / 32;
    const int r = tid;                        // query block i0 + r, TMEM lane r
    const bool live = r < rows;
    const int i = i0 + r;
    uint32_t* scratch = &ctl->scratch[warp][0];
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int32_t* lrow = a.idx + (static_cast<size_t>(bh) * a.nb + (live ? i : i0)) * a.kcap;
    const int lcnt = live ? max(1, min(__ldg(a.cnt + static_cast<size_t>(bh) * a.nb + i), a.kcap)) : 0;
    int cur = 0;
    while (cur < lcnt && __ldg(lrow + cur) < a.pb) ++cur;     // the prefix blocks come first
    unsigned long long* buf =
        a.cand + (static_cast<size_t>(bh) * a.nbv + (live ? i - a.pb : 0)) * kCap;
    int bcnt = 0;
    unsigned long long thr = 0ull;
    float thf = -INFINITY;
    bool ok = true;
    const int last_n = a.N - (a.nb - 1) * kBlock;
    for (int it = 0; it < nblk; ++it) {
      const int j = a.pb + it, b = it & 1;
      if (!sel_wait(&ctl->d_full[b], (it >> 1) & 1, wc)) { ok = false; break; }
      tc_fence_after();
      float x[128];
      const uint32_t dcol = tmem + lane_base + b * 128;
      BSA_TMEM_LD_32F(dcol, x);
      BSA_TMEM_LD_32F(dcol + 32, x + 32);
      BSA_TMEM_LD_32F(dcol + 64, x + 64);
      BSA_TMEM_LD_32F(dcol + 96, x + 96);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&ctl->d_empty[b]);
      bool listed_j = false;
      if (live && cur < lcnt && __ldg(lrow + cur) == j) {
        listed_j = true;
        ++cur;
      }
      if (live && !listed_j) {
        const int nvalid = (j == a.nb - 1) ? last_n : kBlock;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t m = 0;
#pragma unroll
          for (int c = 0; c < 32; ++c) m |= (x[32 * q + c] >= thf) ? (1u << c) : 0u;
          const int lim = nvalid - 32 * q;
          if (lim < 32) m &= lim > 0 ? ((1u << lim) - 1u) : 0u;
          while (m) {
            const int c = __ffs(m) - 1;
            m &= m - 1;
            // x[32q + c] without a dynamic register index
            float xv = x[32 * q];
#pragma unroll
            for (int cc = 1; cc < 32; ++cc) xv = (cc == c) ? x[32 * q + cc] : xv;
            const uint32_t u = static_cast<uint32_t>(j * kBlock + 32 * q + c);
            const unsigned long long key =
                (static_cast<unsigned long long>(orderable_key(xv)) << 32) | static_cast<uint32_t>(~u);
            if (key > thr) buf[bcnt++] = key;
          }
        }
      }
      // compact every full buffer of the warp, one row at a time
      uint32_t need = __ballot_sync(0xffffffffu, live && bcnt > kCap - kBlock);
      while (need) {
        const int L = __ffs(need) - 1;
        need &= need - 1;
        unsigned long long* rb = reinterpret_cast<unsigned long long*>(
            __shfl_sync(0xffffffffu, reinterpret_cast<uintptr_t>(buf), L));
        const int count = __shfl_sync(0xffffffffu, bcnt, L);
        const unsigned long long t = compact_keys<kSlots>(rb, count, a.n_extra, scratch);
        if (lane == L) {
          bcnt = a.n_extra;
          thr = t;
          thf = key_score(t);
        }
      }
    }
    // final: the n_extra largest (or all), written ascending by token
    if (!ok) bcnt = 0;
    for (int L = 0; L < 32; ++L) {
      const int rL = warp * 32 + L;
      if (rL >= rows) break;                   // uniform across the warp
      unsigned long long* rb = reinterpret_cast<unsigned long long*>(
          __shfl_sync(0xffffffffu, reinterpret_cast<uintptr_t>(buf), L));
      int count = __shfl_sync(0xffffffffu, bcnt, L);
      if (count > a.n_extra) {
        compact_keys<kSlots>(rb, count, a.n_extra, scratch);
        count = a.n_extra;
      }
      // tokens into the warp's scratch, then each lane ranks its entries
      for (int p = lane; p < count; p += 32) scratch[p] = ~static_cast<uint32_t>(rb[p]);
      __syncwarp();
      int32_t* orow = a.extra + (static_cast<size_t>(bh) * a.nb + i0 + rL) * a.n_extra;
      for (int p = lane; p < count; p += 32) {
        const uint32_t u = scratch[p];
        int rank = 0;
        for (int q2 = 0; q2 < count; ++q2) rank += scratch[q2] < u ? 1 : 0;
        orow[rank] = static_cast<int32_t>(u);
      }
      for (int p = count + lane; p < a.n_extra; p += 32) orow[p] = -1;
      if (lane == 0) a.ecnt[static_cast<size_t>(bh) * a.nb + i0 + rL] = count;
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kSelMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kSelTmemCols);
  }
}

// ------------------------------------------------------------------ side rows

constexpr int kSumThreads = 128;
constexpr float kDowndateMin = 0.015625f;   // 2^-6

struct SideArgs {
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  const float* anchor;    // [BH, 128]
  const float* kpool;     // [BH, nb, 128]  mean key
  const float* kstat;     // [BH, nb, 128]  fp32 k~ (anchor variant)
  const float* vstat;     // [BH, nb, 128]  fp32 v~ (anchor) / mean v (mean)
  const float* lse_blk;   // [BH, nb]       block LSE at the anchor (anchor variant)
  const int32_t* extra;   // [BH, nb, n_extra] ascending, -1 padded
  const int32_t* ecnt;    // [BH, nb]
  __nv_bfloat16* side_k;  // [BH, nb, scap, 128]
  __nv_bfloat16* side_v;
  float* side_bias;       // [BH, nb, scap]
  int32_t* side_blk;      // [BH, nb, scap]
  int32_t* side_cnt;      // [BH, nb]
  int N, nb, pb, n_extra, scap, variant;
  float scale;
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void load4(const __nv_bfloat16* p, float f[4]) {
  const uint2 w = *reinterpret_cast<const uint2*>(p);
  f[0] = __uint_as_float(w.x << 16);
  f[1] = __uint_as_float(w.x & 0xffff0000u);
  f[2] = __uint_as_float(w.y << 16);
  f[3] = __uint_as_float(w.y & 0xffff0000u);
}

__global__ void __launch_bounds__(kSumThreads) extra_summary_kernel(const SideArgs a) {
  __shared__ int32_t toks[512];
  __shared__ int32_t seg_start[513];
  __shared__ int32_t seg_row[513];
  __shared__ int nseg_s, nrow_s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i = a.pb + blockIdx.x;
  const size_t bh = blockIdx.y;
  const size_t row_id = bh * a.nb + i;
  const int m = max(0, min(__ldg(a.ecnt + row_id), a.n_extra));
  for (int p = tid; p < m; p += kSumThreads) toks[p] = __ldg(a.extra + row_id * a.n_extra + p);
  __syncthreads();
  if (tid == 0) {
    // runs of equal block; a run covering a whole block leaves no row
    int ns = 0, nr = 0;
    for (int p = 0; p < m; ++p) {
      if (p == 0 || (toks[p] >> 7) != (toks[p - 1] >> 7)) {
        seg_start[ns] = p;
        ++ns;
      }
    }
    seg_start[ns] = m;
    for (int s = 0; s < ns; ++s) {
      const int j = toks[seg_start[s]] >> 7;
      const int nj = min(kBlock, a.N - j * kBlock);
      const int e = seg_start[s + 1] - seg_start[s];
      seg_row[s] = (e < nj) ? nr++ : -1;
    }
    nseg_s = ns;
    nrow_s = nr;
  }
  __syncthreads();
  const int nseg = nseg_s, nrow = nrow_s;
  const float* qbar = a.anchor + bh * kDim;
  float qb[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) qb[k] = __ldg(qbar + 4 * lane + k);
  const size_t side_row0 = row_id * a.scap;

  for (int s = warp; s < nseg; s += kSumThreads / 32) {
    const int row = seg_row[s];
    if (row < 0) continue;
    const int p0 = seg_start[s], p1 = seg_start[s + 1];
    const int j = toks[p0] >> 7;
    const int nj = min(kBlock, a.N - j * kBlock);
    const size_t blk = bh * a.nb + j;
    float kn[4], vn[4], Lnew;
    if (a.variant == 0) {
      const float L = __ldg(a.lse_blk + blk);
      float sw = 0.f, swk[4] = {0.f, 0.f, 0.f, 0.f}, swv[4] = {0.f, 0.f, 0.f, 0.f};
      for (int p = p0; p < p1; ++p) {
        const size_t t = bh * a.N + toks[p];
        float kf[4], vf[4];
        load4(a.K + t * kDim + 4 * lane, kf);
        load4(a.V + t * kDim + 4 * lane, vf);
        const float x = warp_sum(qb[0] * kf[0] + qb[1] * kf[1] + qb[2] * kf[2] + qb[3] * kf[3]) *
                        a.scale;
        const float w = expf(x - L);
        sw += w;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          swk[k] = fmaf(w, kf[k], swk[k]);
          swv[k] = fmaf(w, vf[k], swv[k]);
        }
      }
      const float R = 1.f - sw;
      if (R >= kDowndateMin) {
        const float invR = 1.f / R;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          kn[k] = (__ldg(a.kstat + blk * kDim + 4 * lane + k) - swk[k]) * invR;
          vn[k] = (__ldg(a.vstat + blk * kDim + 4 * lane + k) - swv[k]) * invR;
        }
        Lnew = L + logf(R);
      } else {
        // recompute over the remaining rows (max-subtracted sums)
        float mx = -INFINITY, ssum = 0.f, sk[4] = {0.f, 0.f, 0.f, 0.f}, sv[4] = {0.f, 0.f, 0.f, 0.f};
        int q = p0;
        for (int tt = 0; tt < nj; ++tt) {
          const int u = j * kBlock + tt;
          if (q < p1 && toks[q] == u) {
            ++q;
            continue;
          }
          const size_t t = bh * a.N + u;
          float kf[4], vf[4];
          load4(a.K + t * kDim + 4 * lane, kf);
          load4(a.V + t * kDim + 4 * lane, vf);
          const float x = warp_sum(qb[0] * kf[0] + qb[1] * kf[1] + qb[2] * kf[2] + qb[3] * kf[3]) *
                          a.scale;
          const float mn = fmaxf(mx, x);
          const float f = expf(mx - mn), w = expf(x - mn);
          ssum = ssum * f + w;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            sk[k] = fmaf(w, kf[k], sk[k] * f);
            sv[k] = fmaf(w, vf[k], sv[k] * f);
          }
          mx = mn;
        }
        const float inv = 1.f / ssum;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          kn[k] = sk[k] * inv;
          vn[k] = sv[k] * inv;
        }
        Lnew = mx + logf(ssum);
      }
    } else {
      float sk[4] = {0.f, 0.f, 0.f, 0.f}, sv[4] = {0.f, 0.f, 0.f, 0.f};
      for (int p = p0; p < p1; ++p) {
        const size_t t = bh * a.N + toks[p];
        float kf[4], vf[4];
        load4(a.K + t * kDim + 4 * lane, kf);
        load4(a.V + t * kDim + 4 * lane, vf);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          sk[k] += kf[k];
          sv[k] += vf[k];
        }
      }
      const float n = static_cast<float>(nj), rest = static_cast<float>(nj - (p1 - p0));
      const float inv = 1.f / rest;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        kn[k] = (n * __ldg(a.kpool + blk * kDim + 4 * lane + k) - sk[k]) * inv;
        vn[k] = (n * __ldg(a.vstat + blk * kDim + 4 * lane + k) - sv[k]) * inv;
      }
      Lnew = logf(rest);
    }
    // bf16 rows as the MMA will read them; the anchor bias from bf16(k~')
    uint2 kw, vw;
    kw.x = pack_bf16x2(kn[0], kn[1]);
    kw.y = pack_bf16x2(kn[2], kn[3]);
    vw.x = pack_bf16x2(vn[0], vn[1]);
    vw.y = pack_bf16x2(vn[2], vn[3]);
    float bias = Lnew;
    if (a.variant == 0) {
      const float dot = qb[0] * bf16_round(kn[0]) + qb[1] * bf16_round(kn[1]) +
                        qb[2] * bf16_round(kn[2]) + qb[3] * bf16_round(kn[3]);
      bias = Lnew - warp_sum(dot) * a.scale;
    }
    const size_t o = side_row0 + row;
    *reinterpret_cast<uint2*>(a.side_k + o * kDim + 4 * lane) = kw;
    *reinterpret_cast<uint2*>(a.side_v + o * kDim + 4 * lane) = vw;
    if (lane == 0) {
      a.side_bias[o] = bias;
      a.side_blk[o] = j;
    }
  }
  // padding up to the 128-row tile the attention reads: finite zeros, masked
  const int padded = ((nrow + kBlock - 1) / kBlock) * kBlock;
  for (int e = nrow * 32 + tid; e < padded * 32; e += kSumThreads) {
    const size_t o = side_row0 + e / 32;
    const int c = (e % 32) * 4;
    *reinterpret_cast<uint2*>(a.side_k + o * kDim + c) = make_uint2(0, 0);
    *reinterpret_cast<uint2*>(a.side_v + o * kDim + c) = make_uint2(0, 0);
    if (c == 0) {
      a.side_bias[o] = -INFINITY;
      a.side_blk[o] = -1;
    }
  }
  if (tid == 0) a.side_cnt[row_id] = nrow;
}

template <int kCap>
cudaError_t launch_select_extra_t(const Shape& s, const CUtensorMap& tm_k, const SelArgs& a,
                                  cudaStream_t st) {
  constexpr size_t smem = kOffSelCtl + sizeof(SelCtl);
  static std::atomic<bool> attr[64];
  cudaError_t e = once_per_device(attr, [] {
    return cudaFuncSetAttribute(select_extra_kernel<kCap>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (e != cudaSuccess) return e;
  const dim3 grid((s.nbv + kBlock - 1) / kBlock, s.B * s.H);
  select_extra_kernel<kCap><<<grid, kSelThreads, smem, st>>>(tm_k, a);
  return cudaGetLastError();
}

}  // namespace

int extra_cand_cap(int n_extra) { return n_extra <= 256 ? 768 : 1280; }

size_t select_extra_scratch_bytes(const Shape& s, int n_extra) {
  if (n_extra <= 0) return 0;
  return static_cast<size_t>(s.B) * s.H * s.nbv * extra_cand_cap(n_extra) * 8;
}

int extra_side_cap(const Shape& s, int n_extra) {
  const int rows = n_extra < s.nbv ? n_extra : s.nbv;
  return ((rows + kBlock - 1) / kBlock) * kBlock;
}

cudaError_t launch_select_extra(const Shape& s, int n_extra, const CUtensorMap& tm_k,
                                const float* qpool, const int32_t* idx, int kcap,
                                const int32_t* cnt, int32_t* extra, int32_t* ecnt, void* scratch,
                                cudaStream_t st) {
  SelArgs a;
  a.qpool = qpool;
  a.idx = idx;
  a.cnt = cnt;
  a.cand = static_cast<unsigned long long*>(scratch);
  a.extra = extra;
  a.ecnt = ecnt;
  a.dev_status = s.dev_status;
  a.N = s.N;
  a.nb = s.nb;
  a.pb = s.pb;
  a.nbv = s.nbv;
  a.kcap = kcap;
  a.n_extra = n_extra;
  return extra_cand_cap(n_extra) == 768 ? launch_select_extra_t<768>(s, tm_k, a, st)
                                        : launch_select_extra_t<1280>(s, tm_k, a, st);
}

cudaError_t launch_extra_summaries(const Shape& s, int n_extra, const void* K, const void* V,
                                   const float* anchor, const float* kpool, const float* kstat,
                                   const float* vstat, const float* lse_blk, const int32_t* extra,
                                   const int32_t* ecnt, void* side_k, void* side_v,
                                   float* side_bias, int32_t* side_blk, int32_t* side_cnt,
                                   cudaStream_t st) {
  SideArgs a;
  a.K = static_cast<const __nv_bfloat16*>(K);
  a.V = static_cast<const __nv_bfloat16*>(V);
  a.anchor = anchor;
  a.kpool = kpool;
  a.kstat = kstat;
  a.vstat = vstat;
  a.lse_blk = lse_blk;
  a.extra = extra;
  a.ecnt = ecnt;
  a.side_k = static_cast<__nv_bfloat16*>(side_k);
  a.side_v = static_cast<__nv_bfloat16*>(side_v);
  a.side_bias = side_bias;
  a.side_blk = side_blk;
  a.side_cnt = side_cnt;
  a.N = s.N;
  a.nb = s.nb;
  a.pb = s.pb;
  a.n_extra = n_extra;
  a.scap = extra_side_cap(s, n_extra);
  a.variant = s.variant;
  a.scale = 0.088388347648318440550f;
  const dim3 grid(s.nbv, s.B * s.H);
  extra_summary_kernel<<<grid, kSumThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace bsa
