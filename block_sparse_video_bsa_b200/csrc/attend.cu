// Exact branch + compressed branch of block-sparse attention on tcgen05.
//
// Spark-H3 page, section "What Spark-Attn changes": attention is split into
// an exact branch, which computes the highest-ranked key/value blocks in
// full, and a cheap compressed branch for all other blocks.  For one query
// block (128 rows) this kernel streams 128-key tiles:
//   * the listed key blocks idx[0..cnt) (exact branch; the ragged last block
//     is masked by column), then
//   * the summary rows k~_j / v~_j of the video blocks, 128 per tile, with
//     logit + bias_j and the listed / prefix / out-of-range columns masked
//     (compressed branch),
// through one online softmax, so both branches share the running max and sum.
//
// Each CTA runs TWO query blocks ("slots") side by side, so the tensor core
// works on one slot while the other slot's softmax runs.  With a fixed count
// (top-k lists) both slots have the same tile count.  With variable-length
// lists (kVar: the count of each row from cnt) each slot runs its own count;
// the producer and the MMA issuer skip a slot once its tiles are done, and a
// schedule sorted by count inside each head (longest first, heads in order)
// pairs rows of similar length.
// 384 threads in three warpgroups; the two softmax warpgroups raise their
// register budget to 232 and the third lowers its own to 40
// (128*40 + 256*232 = 384*168, the launch allocation):
//   warps 0-3   softmax of slot 0, one thread per query row (TMEM lanes 0-127)
//   warps 4-7   softmax of slot 1
//   warp 8      TMA producer: Q0, Q1, then every K / V tile of both slots in
//               exactly the order the MMA consumes them, through one ring of
//               kRing 32 KB stages (3-D tensor maps [B*H, rows, 128], 128-byte
//               swizzle; rows past the end of a head read as zero).
//   warp 9      TMEM allocator + single-thread tcgen05.mma issuer:
//                 S_s  = Q_s K^T          (A, B from shared memory, K-major)
//                 O_s += P_s V            (A = P from TMEM, B = V MN-major)
//               issue order S0(0) S1(0) | PV0(t) S0(t+1) PV1(t) S1(t+1) | ...
//               MMAs of one thread execute in order, so S_s(t+1) overwrites
//               the TMEM columns of P_s(t) only after PV_s(t) has read them.
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512);
// P_s (bf16, two per 32-bit column) overlays the first 64 columns of S_s.
// Softmax: fp32, base 2 (ex2.approx), lazy O rescale (only when the running
// max grows by more than 2^8), P written with tcgen05.st; epilogue O / l ->
// bf16 and lse.  Every mbarrier wait is bounded (bsa_device.cuh); on expiry
// the CTA records BSA_ERR_TIMEOUT, drains what it issued, frees TMEM and
// returns.
#include "bsa_device.cuh"
#include "bsa_kernels.h"

namespace bsa {

namespace {

constexpr int kThreads = 384;
constexpr uint32_t kSoftmaxRegs = 232, kControlRegs = 40;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kRing = 5;
constexpr uint32_t kTileBytes = 32768;   // 128 x 128 bf16
constexpr uint32_t kSubBytes = 16384;    // 128 rows x 64 bf16 (one 128-byte swizzle atom wide)
constexpr uint32_t kOffQ = 0;            // Q0, Q1
constexpr uint32_t kOffRing = 2 * kTileBytes;
constexpr uint32_t kOffCtl = kOffRing + kRing * kTileBytes;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;
constexpr float kLog2e = 1.4426950408889634074f;
constexpr float kLn2 = 0.69314718055994530942f;
// Lazy rescale threshold (log2 units): p may reach 2^8 before O is rescaled.
constexpr float kRescaleThreshold = 8.0f;

struct Ctl {
  uint64_t full[kRing], empty[kRing];
  uint64_t q_full[2];
  uint64_t s_full[2], p_full[2], o_final[2];
  uint64_t bias_full[2][2], bias_empty[2][2];
  uint64_t fin;
  uint32_t tmem_base;
  int abort_flag;
  int skip;
  alignas(16) float bias_stage[2][2][128];   // [slot][buffer][column]
};
static_assert(kOffCtl + sizeof(Ctl) <= 227 * 1024, "shared memory budget");

struct Args {
  const int32_t* idx;
  const int32_t* cnt;     // list lengths [B*H, nb] (kVar)
  const int32_t* sched;   // video work items, longest list first (kVar)
  const float* bias;
  __nv_bfloat16* O;
  float* lse;
  int* dev_status;
  // extra tokens (kExtra): ascending token lists [B*H, nb, ecap] and their
  // counts, the summary rows of partly extra blocks [B*H, nb, scap] (bias,
  // natural log) and their counts
  const int32_t* extra;
  const int32_t* ecnt;
  const float* side_bias;
  const int32_t* side_cnt;
  int ecap, scap;
  int N, nb, pb, nbv, k_eff, kcap, BH;
  int prefix_ctas;    // CTAs that take dense-prefix query-block pairs
  float scale_log2;   // log2(e) / sqrt(128)
};

// Tensor maps of the extra-token path: K and V as 2-D [B*H*N, 128] with a
// one-row box (row gathers), the side summary rows as [B*H, nb*scap, 128].
struct ExtraMaps {
  CUtensorMap k2, v2, sk, sv;
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtx& wc) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc));
}

// Pair of work items of one CTA: items 2c and 2c+1 of one class (dense-prefix
// query blocks first, then video query blocks, head-major; with a schedule,
// the video items in its order).
struct Pair {
  int bh[2], qi[2];
  bool act1;
};

template <bool kVar>
__device__ __forceinline__ Pair pair_of(int cta, const Args& a) {
  Pair p;
  int base, count, per_head, q0;
  if (cta < a.prefix_ctas) {
    base = 2 * cta;
    count = a.BH * a.pb;
    per_head = a.pb;
    q0 = 0;
  } else {
    base = 2 * (cta - a.prefix_ctas);
    count = a.BH * a.nbv;
    per_head = a.nbv;
    q0 = a.pb;
  }
  p.act1 = base + 1 < count;
  const bool video = cta >= a.prefix_ctas;
  for (int s = 0; s < 2; ++s) {
    int it = min(base + s, count - 1);
    if (kVar && video) it = min(max(__ldg(a.sched + it), 0), count - 1);
    p.bh[s] = it / per_head;
    p.qi[s] = q0 + (it - p.bh[s] * per_head);
  }
  return p;
}

// Is video block j one of the listed blocks (sorted ascending in row[lo, hi))?
__device__ __forceinline__ bool listed(const int32_t* row, int lo, int hi, int j) {
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    const int v = __ldg(row + mid);
    if (v == j) return true;
    if (v < j) lo = mid + 1; else hi = mid;
  }
  return false;
}

// Does the ascending token list row[0..n) hold a token of block j?
__device__ __forceinline__ bool has_token_of(const int32_t* row, int n, int j) {
  int lo = 0, hi = n;
  const int first = j * kBlock;
  while (lo < hi) {   // first position with token >= first
    const int mid = (lo + hi) >> 1;
    if (__ldg(row + mid) < first) lo = mid + 1; else hi = mid;
  }
  return lo < n && __ldg(row + lo) < first + kBlock;
}

// Listed blocks of a video row with a variable-length list, clamped to the
// row's storage (at least one, so the tile loops and the ragged check stay
// inside the row).
__device__ __forceinline__ int list_len(const Args& a, int bh, int qi) {
  const int c = __ldg(a.cnt + static_cast<size_t>(bh) * a.nb + qi);
  return max(1, min(c, min(a.kcap, a.nb)));
}

template <bool kVar, bool kExtra>
__global__ void __launch_bounds__(kThreads, 1)
    attend_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_ks,
                  const __grid_constant__ CUtensorMap tm_vs, const __grid_constant__ ExtraMaps em,
                  const Args a) {
  extern __shared__ __align__(1024) uint8_t sm[];
  Ctl* ctl = reinterpret_cast<Ctl*>(sm + kOffCtl);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // A CTA that starts after another one recorded an expired wait does nothing
  // (decided by one thread so that the whole CTA takes the same branch); so
  // does one whose shared window is not 1024-byte aligned (the swizzled
  // operand layouts need it), after recording the failure.
  if (tid == 0) {
    const bool bad_align = (smem_u32(sm) & 1023u) != 0;
    if (bad_align && a.dev_status) atomicExch(a.dev_status, kErrTimeout);
    ctl->skip = (bad_align || (a.dev_status && *reinterpret_cast<volatile int*>(a.dev_status) != 0))
                    ? 1 : 0;
  }
  __syncthreads();
  if (ctl->skip) return;

  const Pair pr = pair_of<kVar>(blockIdx.x, a);
  const bool video = pr.qi[0] >= a.pb;
  const int u0 = a.pb / kBlock;
  const int sum_tiles = (a.nb + kBlock - 1) / kBlock - u0;
  // Per slot: listed blocks, whether summaries follow, tiles in all.
  int ne0 = video ? a.pb + a.k_eff : a.nb, ne1 = ne0;
  if (kVar && video) {
    ne0 = list_len(a, pr.bh[0], pr.qi[0]);
    ne1 = list_len(a, pr.bh[1], pr.qi[1]);
  }
  const bool hs0 = video && (ne0 - a.pb < a.nbv), hs1 = video && (ne1 - a.pb < a.nbv);
  // Extra tokens (video rows only): ec extra tokens in xe gathered tiles after
  // the listed blocks; sc summary rows of partly extra blocks in st tiles
  // after the global summary tiles.
  int ec0 = 0, ec1 = 0, sc0 = 0, sc1 = 0;
  if (kExtra && video) {
    ec0 = max(0, min(__ldg(a.ecnt + static_cast<size_t>(pr.bh[0]) * a.nb + pr.qi[0]), a.ecap));
    ec1 = max(0, min(__ldg(a.ecnt + static_cast<size_t>(pr.bh[1]) * a.nb + pr.qi[1]), a.ecap));
    sc0 = max(0, min(__ldg(a.side_cnt + static_cast<size_t>(pr.bh[0]) * a.nb + pr.qi[0]), a.scap));
    sc1 = max(0, min(__ldg(a.side_cnt + static_cast<size_t>(pr.bh[1]) * a.nb + pr.qi[1]), a.scap));
  }
  const int xe0 = (ec0 + kBlock - 1) / kBlock, xe1 = (ec1 + kBlock - 1) / kBlock;
  const int st0 = hs0 ? (sc0 + kBlock - 1) / kBlock : 0, st1 = hs1 ? (sc1 + kBlock - 1) / kBlock : 0;
  const int T0 = ne0 + xe0 + (hs0 ? sum_tiles : 0) + st0;
  const int T1 = ne1 + xe1 + (hs1 ? sum_tiles : 0) + st1;
  const int nslots = pr.act1 ? 2 : 1;
  const int steps = (nslots == 2) ? max(T0, T1) : T0;   // tile steps of the CTA
  auto n_exact_of = [&](int s) { return s ? ne1 : ne0; };
  auto tiles_of = [&](int s) { return s ? T1 : T0; };
  auto has_sum_of = [&](int s) { return s ? hs1 : hs0; };
  auto xe_of = [&](int s) { return s ? xe1 : xe0; };
  auto ec_of = [&](int s) { return s ? ec1 : ec0; };
  auto sc_of = [&](int s) { return s ? sc1 : sc0; };

  if (tid == 0) {
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&ctl->full[i], 1);
      mbar_init(&ctl->empty[i], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ctl->q_full[s], 1);
      mbar_init(&ctl->s_full[s], 1);
      mbar_init(&ctl->p_full[s], 128);
      mbar_init(&ctl->o_final[s], 1);
      mbar_init(&ctl->bias_full[s][0], 32);
      mbar_init(&ctl->bias_full[s][1], 32);
      mbar_init(&ctl->bias_empty[s][0], 128);
      mbar_init(&ctl->bias_empty[s][1], 128);
    }
    mbar_init(&ctl->fin, 1);
    ctl->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const WaitCtx wc{&ctl->abort_flag, a.dev_status};

  if (warp >= 8) {
    reg_dealloc<kControlRegs>();
    if (warp == kProducerWarp && (kExtra || lane == 0)) {
    // ---------------------------------------------------------- producer
      // With extra tokens the whole warp runs this loop (each lane issues the
      // row gathers of four rows); otherwise lane 0 alone.  `lead` issues the
      // tile loads and the barrier operations.
      const bool lead = lane == 0;
      auto pwait = [&](uint64_t* bar, uint32_t parity) -> bool {
        if constexpr (kExtra) {
          bool r = true;
          if (lead) r = mbar_wait(bar, parity, wc);
          return __shfl_sync(0xffffffffu, r ? 1 : 0, 0) != 0;
        } else {
          return mbar_wait(bar, parity, wc);
        }
      };
      if (lead) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        for (int s = 0; s < nslots; ++s) {
          mbar_arrive_expect_tx(&ctl->q_full[s], kTileBytes);
          tma_load_3d(sm + kOffQ + s * kTileBytes, &tm_q, &ctl->q_full[s], 0, pr.qi[s] * kBlock,
                      pr.bh[s]);
          tma_load_3d(sm + kOffQ + s * kTileBytes + kSubBytes, &tm_q, &ctl->q_full[s], 64,
                      pr.qi[s] * kBlock, pr.bh[s]);
        }
      }
      int seq = 0;
      bool ok = true;
      // One operand tile (K or V of slot s, tile t) into the next ring stage.
      auto emit = [&](int s, int t, bool is_v) {
        if (!ok) return;
        const int stage = seq % kRing;
        if (seq >= kRing && !pwait(&ctl->empty[stage], ((seq / kRing) - 1) & 1)) {
          ok = false;
          return;
        }
        uint8_t* dst = sm + kOffRing + stage * kTileBytes;
        const int n_exact = n_exact_of(s);
        if (kExtra && t >= n_exact && t < n_exact + xe_of(s)) {
          // 128 extra tokens (padded with the first one) gathered row by row:
          // lane l brings rows 4l..4l+3 of both 64-column halves
          const int x = t - n_exact, ec = ec_of(s);
          const int32_t* erow =
              a.extra + (static_cast<size_t>(pr.bh[s]) * a.nb + pr.qi[s]) * a.ecap;
          const int first = __ldg(erow);
          int rr[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int pos = x * kBlock + 4 * lane + k;
            rr[k] = pr.bh[s] * a.N + (pos < ec ? __ldg(erow + pos) : first);
          }
          if (lead) mbar_arrive_expect_tx(&ctl->full[stage], kTileBytes);
          __syncwarp();
          const CUtensorMap* m = is_v ? &em.v2 : &em.k2;
          tma_gather4(dst + 4 * lane * 128, m, &ctl->full[stage], 0, rr[0], rr[1], rr[2], rr[3]);
          tma_gather4(dst + kSubBytes + 4 * lane * 128, m, &ctl->full[stage], 64, rr[0], rr[1],
                      rr[2], rr[3]);
        } else if (lead) {
          const CUtensorMap* m;
          int row, head = pr.bh[s];
          if (t < n_exact) {
            row = __ldg(a.idx + (static_cast<size_t>(pr.bh[s]) * a.nb + pr.qi[s]) * a.kcap + t) *
                  kBlock;
            m = is_v ? &tm_v : &tm_k;
          } else {
            const int v = t - n_exact - xe_of(s);
            const int gsum = has_sum_of(s) ? sum_tiles : 0;
            if (!kExtra || v < gsum) {
              row = (u0 + v) * kBlock;
              m = is_v ? &tm_vs : &tm_ks;
            } else {
              row = pr.qi[s] * a.scap + (v - gsum) * kBlock;
              m = is_v ? &em.sv : &em.sk;
            }
          }
          mbar_arrive_expect_tx(&ctl->full[stage], kTileBytes);
          tma_load_3d(dst, m, &ctl->full[stage], 0, row, head);
          tma_load_3d(dst + kSubBytes, m, &ctl->full[stage], 64, row, head);
        }
        ++seq;
      };
      for (int s = 0; s < nslots; ++s) emit(s, 0, false);
      for (int t = 0; t < steps && ok; ++t) {
        for (int s = 0; s < nslots; ++s) {
          if (t >= tiles_of(s)) continue;
          emit(s, t, true);
          if (t + 1 < tiles_of(s)) emit(s, t + 1, false);
        }
      }
      // Drain: every issued load has landed before the CTA exits (immediate
      // on the normal path, where the MMA warp already waited for them).
      if (lead) {
        for (int s = 0; s < nslots; ++s) mbar_wait(&ctl->q_full[s], 0, wc);
        for (int k = (seq > kRing ? seq - kRing : 0); k < seq; ++k)
          mbar_wait(&ctl->full[k % kRing], (k / kRing) & 1, wc);
      }
    } else if (warp == kMmaWarp && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
      const uint32_t id_s = idesc_bf16_f32(128, 128, 0);
      const uint32_t id_pv = idesc_bf16_f32(128, 128, 1);
      int seq = 0;
      bool ok = true;
      auto take = [&]() -> uint32_t {   // wait for the next ring stage
        const int stage = seq % kRing;
        if (!mbar_wait(&ctl->full[stage], (seq / kRing) & 1, wc)) ok = false;
        return static_cast<uint32_t>(stage);
      };
      auto release = [&](uint32_t stage) {
        mma_commit(&ctl->empty[stage]);
        ++seq;
      };
      auto issue_s = [&](int s) {
        const uint32_t stage = take();
        if (!ok) return;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sm + kOffQ + s * kTileBytes);
        const uint32_t k_addr = smem_u32(sm + kOffRing + stage * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kSubBytes + (kk & 3) * 32;
          mma_bf16_ss(tmem + kColS + s * 128, smem_desc_sw128(q_addr + off, 16, 1024),
                      smem_desc_sw128(k_addr + off, 16, 1024), id_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&ctl->s_full[s]);
        release(stage);
      };
      auto issue_pv = [&](int s, int t) {
        if (!mbar_wait(&ctl->p_full[s], t & 1, wc)) { ok = false; return; }
        const uint32_t stage = take();
        if (!ok) return;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sm + kOffRing + stage * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          mma_bf16_ts(tmem + kColO + s * 128, tmem + kColS + s * 128 + kk * 8,
                      smem_desc_sw128(v_addr + kk * 2048, kSubBytes, 1024), id_pv,
                      (t > 0 || kk > 0) ? 1u : 0u);
        }
        release(stage);
      };
      for (int s = 0; s < nslots && ok; ++s) {
        if (!mbar_wait(&ctl->q_full[s], 0, wc)) ok = false;
      }
      for (int s = 0; s < nslots && ok; ++s) issue_s(s);
      for (int t = 0; t < steps && ok; ++t) {
        for (int s = 0; s < nslots && ok; ++s) {
          if (t >= tiles_of(s)) continue;
          issue_pv(s, t);
          if (!ok) break;
          if (t + 1 < tiles_of(s)) issue_s(s);
          else mma_commit(&ctl->o_final[s]);
        }
      }
      mma_commit(&ctl->fin);
      mbar_wait(&ctl->fin, 0, wc);
    } else if (warp >= 10 && warp - 10 < nslots && has_sum_of(warp - 10)) {
    // ---------------------------------------------------------- bias stager
      // Warp 10 + s stages, for each summary tile v of slot s, the 128 biases
      // in log2 units with -inf where the column is a listed block, a prefix
      // block or past the last block (listed: binary search of the sorted
      // idx row), double buffered against the slot's softmax warps.
      // With extra tokens, a block that holds some of the row's extra tokens
      // is masked as well (its remaining tokens come as one of the row's side
      // summary rows, staged after the global tiles, -inf past their count).
      const int s = warp - 10;
      const int n_exact = n_exact_of(s);
      const size_t row_id = static_cast<size_t>(pr.bh[s]) * a.nb + pr.qi[s];
      const int32_t* idx_row = a.idx + row_id * a.kcap;
      const float* bias_h = a.bias + static_cast<size_t>(pr.bh[s]) * a.nb;
      const int xe = xe_of(s), ec = ec_of(s), sc = sc_of(s);
      const int gsum = sum_tiles;   // this warp runs only for slots with summaries
      const int32_t* erow = kExtra ? a.extra + row_id * a.ecap : nullptr;
      for (int v = 0; v < tiles_of(s) - n_exact - xe; ++v) {
        if (v >= 2 && !warp_wait(&ctl->bias_empty[s][v & 1], ((v >> 1) - 1) & 1, wc)) break;
        float* dst = &ctl->bias_stage[s][v & 1][0];
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          const int c = lane + 32 * q;
          float b = -INFINITY;
          if (!kExtra || v < gsum) {
            const int j = (u0 + v) * kBlock + c;
            if (j >= a.pb && j < a.nb && !listed(idx_row, a.pb, n_exact, j) &&
                !(kExtra && has_token_of(erow, ec, j)))
              b = __ldg(bias_h + j) * kLog2e;
          } else {
            const int r = (v - gsum) * kBlock + c;
            if (r < sc) b = __ldg(a.side_bias + row_id * a.scap + r) * kLog2e;
          }
          dst[c] = b;
        }
        mbar_arrive(&ctl->bias_full[s][v & 1]);
      }
    }
  } else {
    reg_alloc<kSoftmaxRegs>();
    // ---------------------------------------------------------- softmax
    const int s = warp >> 2;                       // slot
    const int r = tid & 127;                       // query row within the block
    const bool active = s < nslots;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_col = tmem + lane_base + kColS + s * 128;
    const uint32_t o_col = tmem + lane_base + kColO + s * 128;
    const int bh = pr.bh[s], qi = pr.qi[s];
    const int n_exact = n_exact_of(s), T = tiles_of(s);
    const int32_t* idx_row = a.idx + (static_cast<size_t>(bh) * a.nb + qi) * a.kcap;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = active;
    // Only the last listed block can be the ragged last block (lists are
    // ascending and nb-1 is the largest index): find it once.
    int ragged_t = -1, ragged_cols = kBlock;
    if (active && (a.N % kBlock) != 0 && __ldg(idx_row + n_exact - 1) == a.nb - 1) {
      ragged_t = n_exact - 1;
      ragged_cols = a.N - (a.nb - 1) * kBlock;
    }
    const int xe = xe_of(s);
    // valid columns of the last extra tile (the token count need not be a
    // multiple of 128)
    const int extra_last_t = n_exact + xe - 1;
    const int extra_last_cols = ec_of(s) - (xe - 1) * kBlock;
    for (int t = 0; ok && t < T; ++t) {
      const bool exact = t < n_exact + xe;
      const int v = t - n_exact - xe;   // summary tile index when !exact
      if (!warp_wait(&ctl->s_full[s], t & 1, wc)) { ok = false; break; }
      tc_fence_after();
      float x[128];
      BSA_TMEM_LD_32F(s_col, x);
      BSA_TMEM_LD_32F(s_col + 32, x + 32);
      BSA_TMEM_LD_32F(s_col + 64, x + 64);
      BSA_TMEM_LD_32F(s_col + 96, x + 96);
      tmem_wait_ld();

      // Exact tiles keep raw scores (the scale is folded into the exponent's
      // FMA; scale > 0 so max commutes with it); summary tiles become
      // logits in log2 units with the staged bias / mask.
      float2 mul = make_float2(a.scale_log2, a.scale_log2);
      if (exact) {
        if (t == ragged_t) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= ragged_cols) x[c] = -INFINITY;
        }
        if (kExtra && xe > 0 && t == extra_last_t && extra_last_cols < kBlock) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= extra_last_cols) x[c] = -INFINITY;
        }
      } else {
        if (!warp_wait(&ctl->bias_full[s][v & 1], (v >> 1) & 1, wc)) { ok = false; break; }
        const float4* bb4 = reinterpret_cast<const float4*>(&ctl->bias_stage[s][v & 1][0]);
#pragma unroll
        for (int c4 = 0; c4 < 32; ++c4) {
          const float4 b = bb4[c4];
          const float2 y0 = fma2(make_float2(x[4 * c4], x[4 * c4 + 1]), mul, make_float2(b.x, b.y));
          const float2 y1 = fma2(make_float2(x[4 * c4 + 2], x[4 * c4 + 3]), mul, make_float2(b.z, b.w));
          x[4 * c4] = y0.x; x[4 * c4 + 1] = y0.y; x[4 * c4 + 2] = y1.x; x[4 * c4 + 3] = y1.y;
        }
        mbar_arrive(&ctl->bias_empty[s][v & 1]);
        mul = make_float2(1.f, 1.f);
      }
      // row max: 8 independent chains of three-input maxes (64 instructions)
      float mp[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mp[k] = fmaxf(x[k], x[k + 8]);
#pragma unroll
      for (int c = 16; c < 128; c += 16) {
#pragma unroll
        for (int k = 0; k < 8; ++k) mp[k] = fmax3(mp[k], x[c + k], x[c + 8 + k]);
      }
      const float mx = fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]),
                             fmaxf(mp[6], mp[7])) * mul.x;
      const bool need = mx > m_run + kRescaleThreshold;
      const float m_new = need ? mx : m_run;
      const float alpha = need ? fast_exp2(m_run - m_new) : 1.0f;
      // O_s is stable here: PV_s(t-1) was issued before S_s(t) and the MMAs
      // of one thread complete in order.
      if (t > 0 && __any_sync(0xffffffffu, need)) {
        const float2 al2 = make_float2(alpha, alpha);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float o[32];
          BSA_TMEM_LD_32F(o_col + q * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 r2 = mul2(make_float2(o[2 * e], o[2 * e + 1]), al2);
            o[2 * e] = r2.x;
            o[2 * e + 1] = r2.y;
          }
          BSA_TMEM_ST_32(o_col + q * 32, reinterpret_cast<uint32_t*>(o));
        }
      }
      // p = 2^(x * mul - m_new); four packed partial row sums.
      const float2 off = make_float2(-m_new, -m_new);
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float2 y = fma2(make_float2(x[64 * h + 2 * e], x[64 * h + 2 * e + 1]), mul, off);
          const float2 p2 = make_float2(fast_exp2(y.x), fast_exp2(y.y));
          acc[e & 3] = add2(acc[e & 3], p2);
          pk[e] = pack_bf16x2(p2.x, p2.y);
        }
        BSA_TMEM_ST_32(s_col + 32 * h, pk);
      }
      const float2 a01 = add2(acc[0], acc[1]), a23 = add2(acc[2], acc[3]);
      const float2 a4 = add2(a01, a23);
      tmem_wait_st();
      m_run = m_new;
      l_run = l_run * alpha + (a4.x + a4.y);
      tc_fence_before();
      mbar_arrive(&ctl->p_full[s]);
    }
    // -------------------------------------------------------- epilogue
    if (ok && warp_wait(&ctl->o_final[s], 0, wc)) {
      tc_fence_after();
      const int qrow = qi * kBlock + r;
      const bool live = qrow < a.N;
      const float inv_l = 1.f / l_run;
      uint4* orow = reinterpret_cast<uint4*>(a.O + (static_cast<size_t>(bh) * a.N + qrow) * kDim);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float o[32];
        BSA_TMEM_LD_32F(o_col + q * 32, o);
        tmem_wait_ld();
        if (live) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w4[e] = pack_bf16x2(o[v * 8 + 2 * e] * inv_l, o[v * 8 + 2 * e + 1] * inv_l);
            orow[q * 4 + v] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
      }
      if (live && a.lse) a.lse[static_cast<size_t>(bh) * a.N + qrow] = (m_run + __log2f(l_run)) * kLn2;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

__global__ void expired_wait_kernel(int* dev_status, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);   // nothing ever arrives on this barrier
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = globaltimer_ns();
    bool done = false;
    while (!done && globaltimer_ns() - t0 < timeout_ns) done = mbar_try_wait(&bar, 0);
    if (!done) atomicExch(dev_status, kErrTimeout);
  }
}

}  // namespace

namespace {

// Shared setup of both launches: the kernel's shared-memory attribute (once
// per device and instantiation) and the arguments common to both.
template <bool kVar, bool kExtra = false>
cudaError_t attend_attr() {
  constexpr size_t smem = kOffCtl + sizeof(Ctl);
  static std::atomic<bool> attr_set[64];
  return once_per_device(attr_set, [] {
    return cudaFuncSetAttribute(attend_kernel<kVar, kExtra>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
}

Args attend_args(const Shape& s, const int32_t* idx, const float* bias, void* O, float* lse) {
  Args a;
  a.idx = idx;
  a.cnt = nullptr;
  a.sched = nullptr;
  a.extra = nullptr;
  a.ecnt = nullptr;
  a.side_bias = nullptr;
  a.side_cnt = nullptr;
  a.ecap = 0;
  a.scap = 0;
  a.bias = bias;
  a.O = static_cast<__nv_bfloat16*>(O);
  a.lse = lse;
  a.dev_status = s.dev_status;
  a.N = s.N;
  a.nb = s.nb;
  a.pb = s.pb;
  a.nbv = s.nbv;
  a.k_eff = s.k_eff;
  a.kcap = s.kcap;
  a.BH = s.B * s.H;
  a.prefix_ctas = (a.BH * s.pb + 1) / 2;
  a.scale_log2 = kLog2e * 0.088388347648318440550f;
  return a;
}

// ---------------------------------------------------------------- schedule
// Video work items (bh * nbv + qi - pb) ordered head by head and, inside a
// head, by list length, longest first: the two slots of a CTA hold rows of
// similar length, the longest rows of a head start first, and the K/V of only
// one or two heads is in flight at a time (the order of the fixed-count path,
// whose K/V stays in L2).  One CTA per head runs a counting sort of its rows
// in shared memory; the order inside one length follows the shared-memory
// atomics, and no row's result depends on the row it is paired with.
constexpr int kSchedThreads = 512;

__device__ __forceinline__ int item_len(const int32_t* cnt, int it, int nbv, int nb, int pb,
                                        int kcap) {
  const int bh = it / nbv, qi = pb + (it - bh * nbv);
  const int c = __ldg(cnt + static_cast<size_t>(bh) * nb + qi);
  return max(1, min(c, min(kcap, nb)));
}

__global__ void __launch_bounds__(kSchedThreads)
    head_schedule_kernel(const int32_t* __restrict__ cnt, int nbv, int nb, int pb, int kcap,
                         int32_t* __restrict__ sched) {
  extern __shared__ int sm_sched[];
  int* hist = sm_sched;                  // [nb + 1] rows per length
  int* cur = sm_sched + (nb + 1);        // [nb + 1] first position of each length
  __shared__ int part[kSchedThreads];
  const int tid = threadIdx.x, nbins = nb + 1;
  const int base = blockIdx.x * nbv;     // this head's items
  for (int b = tid; b < nbins; b += kSchedThreads) hist[b] = 0;
  __syncthreads();
  for (int r = tid; r < nbv; r += kSchedThreads)
    atomicAdd(&hist[item_len(cnt, base + r, nbv, nb, pb, kcap)], 1);
  __syncthreads();
  // cur[b] = rows with a longer list: thread t scans a contiguous run of the
  // reversed bins, then the run totals are scanned across the block.
  const int per = (nbins + kSchedThreads - 1) / kSchedThreads;
  const int r0 = min(nbins, tid * per), r1 = min(nbins, r0 + per);
  int run = 0;
  for (int r = r0; r < r1; ++r) run += hist[nb - r];
  part[tid] = run;
  __syncthreads();
  for (int off = 1; off < kSchedThreads; off <<= 1) {      // inclusive scan of part
    const int v = tid >= off ? part[tid - off] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int acc = part[tid] - run;                                // exclusive prefix of the run
  for (int r = r0; r < r1; ++r) {
    cur[nb - r] = acc;
    acc += hist[nb - r];
  }
  __syncthreads();
  for (int r = tid; r < nbv; r += kSchedThreads) {
    const int pos = atomicAdd(&cur[item_len(cnt, base + r, nbv, nb, pb, kcap)], 1);
    if (pos >= 0 && pos < nbv) sched[base + pos] = base + r;
  }
}

}  // namespace

cudaError_t launch_attend(const Shape& s, const AttendMaps& maps, const int32_t* idx,
                          const int32_t* cnt, const float* bias, void* O, float* lse,
                          cudaStream_t st) {
  // Tile counts follow from (pb, k_eff, nb): bsa_select lists pb + k_eff
  // blocks for every video query block and all nb for a prefix block.
  (void)cnt;
  cudaError_t e = attend_attr<false>();
  if (e != cudaSuccess) return e;
  const Args a = attend_args(s, idx, bias, O, lse);
  const int grid = a.prefix_ctas + (a.BH * s.nbv + 1) / 2;
  const ExtraMaps none{};
  attend_kernel<false, false><<<grid, kThreads, kOffCtl + sizeof(Ctl), st>>>(
      maps.q, maps.k, maps.v, maps.ks, maps.vs, none, a);
  return cudaGetLastError();
}

size_t attend_lists_scratch_bytes(const Shape& s) {
  return static_cast<size_t>(s.B) * s.H * s.nbv * 4;
}

cudaError_t launch_attend_lists(const Shape& s, const AttendMaps& maps, const int32_t* idx,
                                int kcap, const int32_t* cnt, const float* bias, void* O,
                                float* lse, void* scratch, cudaStream_t st) {
  cudaError_t e = attend_attr<true>();
  if (e != cudaSuccess) return e;
  const size_t smem_sched = 2 * (static_cast<size_t>(s.nb) + 1) * sizeof(int);
  static std::atomic<bool> sched_attr[64];
  e = once_per_device(sched_attr, [] {
    const int max_dyn = 2 * (16384 + 1) * static_cast<int>(sizeof(int));
    return cudaFuncSetAttribute(head_schedule_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                max_dyn);
  });
  if (e != cudaSuccess) return e;
  int32_t* sched = static_cast<int32_t*>(scratch);
  head_schedule_kernel<<<s.B * s.H, kSchedThreads, smem_sched, st>>>(cnt, s.nbv, s.nb, s.pb, kcap,
                                                                     sched);
  Args a = attend_args(s, idx, bias, O, lse);
  a.cnt = cnt;
  a.sched = sched;
  a.kcap = kcap;
  const int grid = a.prefix_ctas + (a.BH * s.nbv + 1) / 2;
  const ExtraMaps none{};
  attend_kernel<true, false><<<grid, kThreads, kOffCtl + sizeof(Ctl), st>>>(
      maps.q, maps.k, maps.v, maps.ks, maps.vs, none, a);
  return cudaGetLastError();
}

cudaError_t launch_attend_extra(const Shape& s, const AttendMaps& maps,
                                const AttendExtraMaps& xmaps, const int32_t* idx,
                                const int32_t* extra, const int32_t* ecnt, int ecap,
                                const float* bias, const float* side_bias, const int32_t* side_cnt,
                                int scap, void* O, float* lse, cudaStream_t st) {
  cudaError_t e = attend_attr<false, true>();
  if (e != cudaSuccess) return e;
  Args a = attend_args(s, idx, bias, O, lse);
  a.extra = extra;
  a.ecnt = ecnt;
  a.ecap = ecap;
  a.side_bias = side_bias;
  a.side_cnt = side_cnt;
  a.scap = scap;
  ExtraMaps em;
  em.k2 = xmaps.k2;
  em.v2 = xmaps.v2;
  em.sk = xmaps.sk;
  em.sv = xmaps.sv;
  const int grid = a.prefix_ctas + (a.BH * s.nbv + 1) / 2;
  attend_kernel<false, true><<<grid, kThreads, kOffCtl + sizeof(Ctl), st>>>(
      maps.q, maps.k, maps.v, maps.ks, maps.vs, em, a);
  return cudaGetLastError();
}

cudaError_t launch_expired_wait(int32_t* dev_status, uint64_t timeout_ns, cudaStream_t st) {
  expired_wait_kernel<<<1, 32, 0, st>>>(dev_status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace bsa
