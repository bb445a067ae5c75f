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
//                        (four buffers).  Two threads per query block, one
//                        per half of each key block's 128 tokens, each keep a
//                        running threshold and append the candidates above
//                        it to their own buffer in global memory as 64-bit
//                        keys (order-preserving score bits << 32 | ~token, so
//                        a larger key is a higher score, then a lower index);
//                        when a buffer fills, the warp compacts it to the
//                        n_extra largest keys (bitwise binary search with
//                        warp-wide counts) and raises the threshold to the
//                        smallest kept key.
//  extra_finish_kernel   one warp per query block: the n_extra largest keys
//                        of its two buffers (each holds the n_extra largest of
//                        its half, so their union holds the row's), written
//                        as tokens in ascending order.
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

// warps 0-7 select (warp w: TMEM lanes 32 (w % 4) .., token half w / 4),
// warp 8 producer, warp 9 MMA
constexpr int kSelWarps = 8;
constexpr int kSelThreads = 32 * kSelWarps + 64;
constexpr int kSelProducerWarp = kSelWarps;
constexpr int kSelMmaWarp = kSelWarps + 1;
constexpr int kSelRing = 4;
constexpr uint32_t kTileB = 32768;   // 128 x 128 bf16
constexpr uint32_t kHalfB = 16384;   // 128 rows x 64 bf16 (one 128-byte swizzle atom wide)
constexpr uint32_t kOffAhi = 0;
constexpr uint32_t kOffAlo = kTileB;
constexpr uint32_t kOffRingB = 2 * kTileB;
constexpr uint32_t kOffSelCtl = kOffRingB + kSelRing * kTileB;
constexpr uint32_t kSelTmemCols = 512;
constexpr int kDBuf = 4;   // score buffers in TMEM (the selection warps may drift apart)

struct SelCtl {
  uint64_t full[kSelRing], empty[kSelRing];
  uint64_t d_full[kDBuf], d_empty[kDBuf];
  uint64_t fin;
  uint32_t tmem_base;
  int abort_flag;
  int skip;
  // each (token half, row) thread's threshold key, read by the row's other
  // thread: the n_extra-th largest key of either half bounds the row's from below
  unsigned long long rthr[2][kBlock];
  // per selection warp: the 32 scores of a column group of every lane, [column][lane],
  // read back by the lanes' appends; the compaction's 64-key scratch in between
  alignas(16) float xs[kSelWarps][32][32];
};
static_assert(kOffSelCtl + sizeof(SelCtl) <= 227 * 1024, "shared memory budget");

struct SelArgs {
  const float* qpool;          // [BH, nb, 128]
  const int32_t* idx;          // [BH, nb, kcap]
  const int32_t* cnt;          // [BH, nb]
  unsigned long long* cand;    // [BH * nbv, 2, kCap] candidate buffers (two token halves)
  int32_t* bcnt;               // [BH * nbv, 2] keys left in each buffer
  int rows_v;                  // BH * nbv
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
// smallest kept key.  The target-th largest key is found by a bitwise binary
// search with warp-wide counts (no shared-memory atomics): first on the score
// half of the keys, then, when several keys share that score, on the token
// half among them (a single one is found by a minimum).  Requires
// 1 <= target <= count <= 32 * kSlots.
// Exclusive prefix sum of v over the lanes of the warp.
__device__ __forceinline__ int lane_prefix(int v, int lane) {
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x - v;
}

// The search over the score halves counts all keys only until the range
// [th, th + 2^b) known to hold the target-th largest score holds at most 64
// keys; those go to `scratch` (64 keys, the warp's own), two per lane, and the
// search (and the token-half search among equal scores) finishes on them.
template <int kSlots>
__device__ unsigned long long compact_keys(unsigned long long* buf, int count, int target,
                                           unsigned long long* scratch) {
  const int lane = threadIdx.x & 31;
  __syncwarp();   // the owner's appends are visible to every lane
  uint32_t hi[kSlots], lo[kSlots];
#pragma unroll
  for (int k = 0; k < kSlots; ++k) {
    const int p = lane + 32 * k;
    const unsigned long long e = p < count ? buf[p] : 0ull;
    hi[k] = static_cast<uint32_t>(e >> 32);
    lo[k] = static_cast<uint32_t>(e);
  }
  __syncwarp();
  // largest T_hi with #{hi >= T_hi} >= target (empty slots have hi = 0 and
  // every real key has hi > 0)
  uint32_t th = 0;
  int above = 0, at_least = count;   // keys with hi at or above the range's top / >= th
  int b = 31;
  for (; b >= 0; --b) {
    const uint32_t cand = th | (1u << b);
    int c4[4] = {0, 0, 0, 0};   // independent partial counts
#pragma unroll
    for (int k = 0; k < kSlots; ++k) c4[k & 3] += hi[k] >= cand ? 1 : 0;
    const int c =
        static_cast<int>(__reduce_add_sync(0xffffffffu, (c4[0] + c4[1]) + (c4[2] + c4[3])));
    if (c >= target) {
      th = cand;
      at_least = c;
    } else {
      above = c;
    }
    if (at_least - above <= 64) break;
  }
  int gt, eq;
  uint32_t tl;
  if (b > 0) {
    // the range's keys (at most 64) to the scratch, two per lane
    const uint32_t width = 1u << b;
    int own = 0;
#pragma unroll
    for (int k = 0; k < kSlots; ++k) own += (hi[k] != 0u && hi[k] - th < width) ? 1 : 0;
    int pos = lane_prefix(own, lane);
#pragma unroll
    for (int k = 0; k < kSlots; ++k)
      if (hi[k] != 0u && hi[k] - th < width)
        scratch[pos++] = (static_cast<unsigned long long>(hi[k]) << 32) | lo[k];
    __syncwarp();
    const int nc = at_least - above;
    const unsigned long long e0 = lane < nc ? scratch[lane] : 0ull;
    const unsigned long long e1 = lane + 32 < nc ? scratch[lane + 32] : 0ull;
    __syncwarp();
    const uint32_t h0 = static_cast<uint32_t>(e0 >> 32), h1 = static_cast<uint32_t>(e1 >> 32);
    const uint32_t l0 = static_cast<uint32_t>(e0), l1 = static_cast<uint32_t>(e1);
    // every candidate lies below the keys counted in `above`
    for (--b; b >= 0; --b) {
      const uint32_t cand = th | (1u << b);
      const int c = above + static_cast<int>(__reduce_add_sync(
                                0xffffffffu, (h0 >= cand ? 1 : 0) + (h1 >= cand ? 1 : 0)));
      if (c >= target) th = cand;
    }
    gt = above + static_cast<int>(
                     __reduce_add_sync(0xffffffffu, (h0 > th ? 1 : 0) + (h1 > th ? 1 : 0)));
    const bool q0 = lane < nc && h0 == th, q1 = lane + 32 < nc && h1 == th;
    eq = static_cast<int>(__reduce_add_sync(0xffffffffu, (q0 ? 1 : 0) + (q1 ? 1 : 0)));
    const int need = target - gt;   // 1 <= need <= eq
    if (need == eq) {
      tl = __reduce_min_sync(0xffffffffu, min(q0 ? l0 : 0xffffffffu, q1 ? l1 : 0xffffffffu));
    } else {   // several keys share the score: the need-th largest token half among them
      tl = 0;
      for (int bb = 31; bb >= 0; --bb) {
        const uint32_t cand = tl | (1u << bb);
        const int c = static_cast<int>(__reduce_add_sync(
            0xffffffffu, ((q0 && l0 >= cand) ? 1 : 0) + ((q1 && l1 >= cand) ? 1 : 0)));
        if (c >= need) tl = cand;
      }
    }
  } else {
    int g = 0, q = 0;
    uint32_t eq_min = 0xffffffffu;
#pragma unroll
    for (int k = 0; k < kSlots; ++k) {
      g += hi[k] > th ? 1 : 0;
      if (hi[k] == th) {
        ++q;
        eq_min = min(eq_min, lo[k]);
      }
    }
    gt = static_cast<int>(__reduce_add_sync(0xffffffffu, g));
    eq = static_cast<int>(__reduce_add_sync(0xffffffffu, q));
    const int need = target - gt;   // 1 <= need <= eq
    if (need == eq) {
      tl = __reduce_min_sync(0xffffffffu, eq_min);
    } else {   // several keys share the score: the need-th largest token half among them
      tl = 0;
      for (int bb = 31; bb >= 0; --bb) {
        const uint32_t cand = tl | (1u << bb);
        int c = 0;
#pragma unroll
        for (int k = 0; k < kSlots; ++k) c += (hi[k] == th && lo[k] >= cand) ? 1 : 0;
        if (static_cast<int>(__reduce_add_sync(0xffffffffu, c)) >= need) tl = cand;
      }
    }
  }
  const unsigned long long T = (static_cast<unsigned long long>(th) << 32) | tl;
  int out = 0;
#pragma unroll
  for (int k = 0; k < kSlots; ++k) {
    const unsigned long long e = (static_cast<unsigned long long>(hi[k]) << 32) | lo[k];
    const bool keep = hi[k] != 0u && e >= T;
    const uint32_t m = __ballot_sync(0xffffffffu, keep);
    if (keep) buf[out + __popc(m & ((1u << lane) - 1u))] = e;
    out += __popc(m);
  }
  __syncwarp();
  return T;
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
    for (int b = 0; b < kDBuf; ++b) {
      mbar_init(&ctl->d_full[b], 1);
      mbar_init(&ctl->d_empty[b], 32 * kSelWarps);
    }
    mbar_init(&ctl->fin, 1);
    for (int e = 0; e < 2 * kBlock; ++e) ctl->rthr[e >> 7][e & (kBlock - 1)] = 0ull;
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
        const int stage = it % kSelRing, b = it % kDBuf;
        if (!mbar_wait(&ctl->full[stage], (it / kSelRing) & 1, wc)) { ok = false; break; }
        if (it >= kDBuf && !mbar_wait(&ctl->d_empty[b], ((it / kDBuf) - 1) & 1, wc)) {
          ok = false;
          break;
        }
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
    const int half = warp >> 2;               // tokens 64 half .. 64 half + 63 of each key block
    const int r = (warp & 3) * 32 + lane;     // query block i0 + r, TMEM lane r
    const bool live = r < rows;
    const int i = i0 + r;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int32_t* lrow = a.idx + (static_cast<size_t>(bh) * a.nb + (live ? i : i0)) * a.kcap;
    const int lcnt = live ? max(1, min(__ldg(a.cnt + static_cast<size_t>(bh) * a.nb + i), a.kcap)) : 0;
    int cur = 0;
    while (cur < lcnt && __ldg(lrow + cur) < a.pb) ++cur;     // the prefix blocks come first
    const size_t brow = (static_cast<size_t>(bh) * a.nbv + (live ? i - a.pb : 0)) * 2 + half;
    unsigned long long* buf = a.cand + brow * kCap;
    int bcnt = 0;
    unsigned long long thr = 0ull;
    float thf = -INFINITY;
    bool ok = true;
    float (*xsw)[32] = ctl->xs[warp];
    const int last_n = a.N - (a.nb - 1) * kBlock;
    for (int it = 0; it < nblk; ++it) {
      const int j = a.pb + it, b = it % kDBuf;
      if (!sel_wait(&ctl->d_full[b], (it / kDBuf) & 1, wc)) { ok = false; break; }
      tc_fence_after();
      float x[64];
      const uint32_t dcol = tmem + lane_base + b * 128 + 64 * half;
      BSA_TMEM_LD_32F(dcol, x);
      BSA_TMEM_LD_32F(dcol + 32, x + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&ctl->d_empty[b]);
      if (live) {   // the other half's threshold, when higher (a stale one is merely looser)
        const unsigned long long o =
            *reinterpret_cast<volatile unsigned long long*>(&ctl->rthr[half ^ 1][r]);
        if (o > thr) {
          thr = o;
          thf = key_score(o);
        }
      }
      bool listed_j = false;
      if (live && cur < lcnt && __ldg(lrow + cur) == j) {
        listed_j = true;
        ++cur;
      }
      const bool scan = live && !listed_j;
      const int nvalid = (j == a.nb - 1) ? last_n : kBlock;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int c0 = 64 * half + 32 * q;    // first token of the group within the block
        uint32_t m = 0;
        if (scan) {
#pragma unroll
          for (int c = 0; c < 32; ++c) m |= (x[32 * q + c] >= thf) ? (1u << c) : 0u;
          const int lim = nvalid - c0;
          if (lim < 32) m &= lim > 0 ? ((1u << lim) - 1u) : 0u;
        }
        // every lane walks its own set bits: the lanes append together, each
        // reading its score back from the warp's copy of the group
        if (__any_sync(0xffffffffu, m != 0)) {
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 32; ++c) xsw[c][lane] = x[32 * q + c];
          __syncwarp();
        }
        while (m) {
          const int c = __ffs(m) - 1;
          m &= m - 1;
          const float xv = xsw[c][lane];
          const uint32_t u = static_cast<uint32_t>(j * kBlock + c0 + c);
          const unsigned long long key =
              (static_cast<unsigned long long>(orderable_key(xv)) << 32) |
              static_cast<uint32_t>(~u);
          if (key > thr) buf[bcnt++] = key;
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
        const unsigned long long t = compact_keys<kSlots>(
            rb, count, a.n_extra, reinterpret_cast<unsigned long long*>(&xsw[0][0]));
        if (lane == L) {
          bcnt = a.n_extra;
          if (t > thr) {
            thr = t;
            thf = key_score(t);
          }
          *reinterpret_cast<volatile unsigned long long*>(&ctl->rthr[half][r]) = thr;
        }
      }
    }
    // the buffer's fill count goes to the finishing kernel, which keeps the
    // n_extra largest keys and writes them ascending by token
    if (live) a.bcnt[brow] = ok ? bcnt : 0;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kSelMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kSelTmemCols);
  }
}

// One warp per video query block: the n_extra largest keys of its two
// buffers (compactions when more are left), written as tokens in ascending order
// (each lane ranks its entries by counting smaller tokens in the warp's
// shared buffer, four per 16-byte read), -1 padded; ecnt = their count.
constexpr int kFinThreads = 256;

template <int kCap>
__global__ void __launch_bounds__(kFinThreads) extra_finish_kernel(const SelArgs a) {
  __shared__ alignas(16) uint32_t sbuf[kFinThreads / 32][512 + 4];   // n_extra <= 512
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rowv = blockIdx.x * (kFinThreads / 32) + warp;   // video row over all heads
  if (rowv >= a.rows_v) return;                               // whole warp
  const int bh = rowv / a.nbv, i = a.pb + rowv % a.nbv;
  unsigned long long* rb = a.cand + static_cast<size_t>(rowv) * 2 * kCap;
  unsigned long long* rb1 = rb + kCap;
  uint32_t* tok = sbuf[warp];
  // each half's buffer down to its n_extra largest keys, the second appended
  // to the first (2 n_extra <= kCap), then the n_extra largest of the union
  int count = max(0, min(__ldg(a.bcnt + 2 * rowv), kCap));
  int count1 = max(0, min(__ldg(a.bcnt + 2 * rowv + 1), kCap));
  if (count > a.n_extra) {
    compact_keys<kCap / 32>(rb, count, a.n_extra, reinterpret_cast<unsigned long long*>(tok));
    count = a.n_extra;
  }
  if (count1 > a.n_extra) {
    compact_keys<kCap / 32>(rb1, count1, a.n_extra, reinterpret_cast<unsigned long long*>(tok));
    count1 = a.n_extra;
  }
  for (int p = lane; p < count1; p += 32) rb[count + p] = rb1[p];
  count += count1;
  if (count > a.n_extra) {
    compact_keys<kCap / 32>(rb, count, a.n_extra, reinterpret_cast<unsigned long long*>(tok));
    count = a.n_extra;
  }
  for (int p = lane; p < count; p += 32) tok[p] = ~static_cast<uint32_t>(rb[p]);
  for (int p = count + lane; p < ((count + 3) & ~3); p += 32) tok[p] = 0xffffffffu;
  __syncwarp();
  int32_t* orow = a.extra + (static_cast<size_t>(bh) * a.nb + i) * a.n_extra;
  const uint4* t4 = reinterpret_cast<const uint4*>(tok);
  for (int p = lane; p < count; p += 32) {
    const uint32_t u = tok[p];
    int r4[4] = {0, 0, 0, 0};
    for (int q4 = 0; q4 < (count + 3) / 4; ++q4) {
      const uint4 t = t4[q4];
      r4[0] += t.x < u ? 1 : 0;
      r4[1] += t.y < u ? 1 : 0;
      r4[2] += t.z < u ? 1 : 0;
      r4[3] += t.w < u ? 1 : 0;
    }
    orow[(r4[0] + r4[1]) + (r4[2] + r4[3])] = static_cast<int32_t>(u);
  }
  for (int p = count + lane; p < a.n_extra; p += 32) orow[p] = -1;
  if (lane == 0) a.ecnt[static_cast<size_t>(bh) * a.nb + i] = count;
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


__device__ __forceinline__ void bf16x4_to_f32(uint2 w, float f[4]) {
  f[0] = __uint_as_float(w.x << 16);
  f[1] = __uint_as_float(w.x & 0xffff0000u);
  f[2] = __uint_as_float(w.y << 16);
  f[3] = __uint_as_float(w.y & 0xffff0000u);
}

// One CTA (4 warps) per video query block; each warp takes runs of tokens of
// one block (lane l: dimensions 4l..4l+3), gathering each token's K and V row
// once: its anchor logit (a warp sum), its weight and its share of the sums.
__global__ void __launch_bounds__(kSumThreads, 8) extra_summary_kernel(const SideArgs a) {
  __shared__ int32_t toks[512];
  __shared__ int32_t seg_start[513];
  __shared__ int32_t seg_row[513];
  __shared__ int nseg_s, nrow_s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i = a.pb + blockIdx.x;
  const size_t bh = blockIdx.y;
  const size_t row_id = bh * a.nb + i;
  const int m_in = max(0, min(__ldg(a.ecnt + row_id), a.n_extra));
  const bool anchor_variant = a.variant == 0;
  for (int p = tid; p < m_in; p += kSumThreads) toks[p] = __ldg(a.extra + row_id * a.n_extra + p);
  __syncthreads();
  if (tid == 0) {
    // the list is used up to its first token that is not a video token or
    // not above its predecessor (a valid list has none), so every row read
    // below lies inside the head
    int m = 0;
    while (m < m_in && toks[m] >= a.pb * kBlock && toks[m] < a.N &&
           (m == 0 || toks[m] > toks[m - 1]))
      ++m;
    // runs of equal block; a run covering a whole block leaves no row
    int ns = 0, nr = 0;
    for (int p = 0; p < m; ++p) {
      if (p == 0 || (toks[p] >> 7) != (toks[p - 1] >> 7)) seg_start[ns++] = p;
    }
    seg_start[ns] = m;
    for (int s = 0; s < ns; ++s) {
      const int j = toks[seg_start[s]] >> 7;
      const int nj = min(kBlock, a.N - j * kBlock);
      seg_row[s] = (seg_start[s + 1] - seg_start[s] < nj) ? nr++ : -1;
    }
    nseg_s = ns;
    nrow_s = nr;
  }
  __syncthreads();
  const int nseg = nseg_s, nrow = nrow_s;
  const size_t side_row0 = row_id * a.scap;
  float q4[4] = {0.f, 0.f, 0.f, 0.f};
  if (anchor_variant) {
    const float4 t = __ldg(reinterpret_cast<const float4*>(a.anchor + bh * kDim) + lane);
    q4[0] = t.x; q4[1] = t.y; q4[2] = t.z; q4[3] = t.w;
  }
  auto logit = [&](const float kf[4]) {
    return warp_sum(q4[0] * kf[0] + q4[1] * kf[1] + q4[2] * kf[2] + q4[3] * kf[3]) * a.scale;
  };

  for (int s = warp; s < nseg; s += kSumThreads / 32) {
    const int row = seg_row[s];
    if (row < 0) continue;
    const int p0 = seg_start[s], p1 = seg_start[s + 1];
    const int j = toks[p0] >> 7;
    const int nj = min(kBlock, a.N - j * kBlock);
    const size_t blk = bh * a.nb + j;
    float kn[4], vn[4], Lnew;
    if (anchor_variant) {
      const float L = __ldg(a.lse_blk + blk);
      float sw = 0.f, swk[4] = {0.f, 0.f, 0.f, 0.f}, swv[4] = {0.f, 0.f, 0.f, 0.f};
      for (int p = p0; p < p1; ++p) {
        const size_t t = bh * a.N + toks[p];
        float kf[4], vf[4];
        bf16x4_to_f32(*reinterpret_cast<const uint2*>(a.K + t * kDim + 4 * lane), kf);
        bf16x4_to_f32(*reinterpret_cast<const uint2*>(a.V + t * kDim + 4 * lane), vf);
        const float w = expf(logit(kf) - L);
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
        const float4 ks4 = __ldg(reinterpret_cast<const float4*>(a.kstat + blk * kDim) + lane);
        const float4 vs4 = __ldg(reinterpret_cast<const float4*>(a.vstat + blk * kDim) + lane);
        kn[0] = (ks4.x - swk[0]) * invR; kn[1] = (ks4.y - swk[1]) * invR;
        kn[2] = (ks4.z - swk[2]) * invR; kn[3] = (ks4.w - swk[3]) * invR;
        vn[0] = (vs4.x - swv[0]) * invR; vn[1] = (vs4.y - swv[1]) * invR;
        vn[2] = (vs4.z - swv[2]) * invR; vn[3] = (vs4.w - swv[3]) * invR;
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
          bf16x4_to_f32(*reinterpret_cast<const uint2*>(a.K + t * kDim + 4 * lane), kf);
          bf16x4_to_f32(*reinterpret_cast<const uint2*>(a.V + t * kDim + 4 * lane), vf);
          const float x = logit(kf);
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
        bf16x4_to_f32(*reinterpret_cast<const uint2*>(a.K + t * kDim + 4 * lane), kf);
        bf16x4_to_f32(*reinterpret_cast<const uint2*>(a.V + t * kDim + 4 * lane), vf);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          sk[k] += kf[k];
          sv[k] += vf[k];
        }
      }
      const float n = static_cast<float>(nj), rest = static_cast<float>(nj - (p1 - p0));
      const float4 kp4 = __ldg(reinterpret_cast<const float4*>(a.kpool + blk * kDim) + lane);
      const float4 vs4 = __ldg(reinterpret_cast<const float4*>(a.vstat + blk * kDim) + lane);
      kn[0] = (n * kp4.x - sk[0]) / rest; kn[1] = (n * kp4.y - sk[1]) / rest;
      kn[2] = (n * kp4.z - sk[2]) / rest; kn[3] = (n * kp4.w - sk[3]) / rest;
      vn[0] = (n * vs4.x - sv[0]) / rest; vn[1] = (n * vs4.y - sv[1]) / rest;
      vn[2] = (n * vs4.z - sv[2]) / rest; vn[3] = (n * vs4.w - sv[3]) / rest;
      Lnew = logf(rest);
    }
    // bf16 rows as the MMA will read them; the anchor bias from bf16(k~')
    uint2 kw, vw;
    kw.x = pack_bf16x2(kn[0], kn[1]);
    kw.y = pack_bf16x2(kn[2], kn[3]);
    vw.x = pack_bf16x2(vn[0], vn[1]);
    vw.y = pack_bf16x2(vn[2], vn[3]);
    float bias = Lnew;
    if (anchor_variant) {
      float kb[4];
      bf16x4_to_f32(kw, kb);
      bias = Lnew - logit(kb);
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
  const int fgrid = (a.rows_v + kFinThreads / 32 - 1) / (kFinThreads / 32);
  extra_finish_kernel<kCap><<<fgrid, kFinThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

// Candidate keys per query block: 768 up to 256 extra tokens (measured at
// 256 on 768p-5s / 2K-5s: 4.00 / 17.1 ms against 4.20 / 18.4 with 1280 and
// 4.57 / 18.3 with 512), 2048 above.
int extra_cand_cap(int n_extra) { return n_extra <= 256 ? 768 : 2048; }

size_t select_extra_scratch_bytes(const Shape& s, int n_extra) {
  if (n_extra <= 0) return 0;
  const size_t bufs = static_cast<size_t>(s.B) * s.H * s.nbv * 2;   // two per video query block
  return bufs * extra_cand_cap(n_extra) * 8 + bufs * 4;   // buffers, then their fill counts
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
  a.rows_v = s.B * s.H * s.nbv;
  a.bcnt = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(scratch) +
                                      static_cast<size_t>(a.rows_v) * 2 *
                                          extra_cand_cap(n_extra) * 8);
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
                                        : launch_select_extra_t<2048>(s, tm_k, a, st);
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
