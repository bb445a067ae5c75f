// Exact branch + compressed branch of block-sparse attention with FP8 (e4m3)
// operands on tcgen05 (kind::f8f6f4).
//
// Same method and work decomposition as attend.cu (Spark-H3 page, section
// "What Spark-Attn changes": an exact branch over the top-ranked key/value
// blocks and a compressed branch over one summary row per other block, in
// one online softmax); the operands are the per-group e4m3 codes written by
// quant_fp8.cu (the pages' quantised sparse kernel, "H3 Sparse Attention",
// comfy.icu WAS node, section "What it actually does"; format and scaling are
// this library's reading).
//
// What differs from the bf16 kernel:
//   * every tile is one 128 x 128-byte box (16 KB): Q_s, K and the summary
//     keys row-major, V and the summary values dimension-major per group, so
//     both MMAs read K-major operands; the ring holds kRing = 12 tiles;
//   * S_s = Q_s K^T is 4 MMAs of K = 32; O_s += P_s V is 4 MMAs with P_s in
//     TMEM as four e4m3 per 32-bit column (32 columns);
//   * logits scale by log2(e)/sqrt(d) * s_q * s_k (per query block and per
//     key block or summary tile); the softmax numerators p enter P as
//     e4m3(p * s_v / v_ref) with v_ref the largest value scale of the head, so
//     O = v_ref * (sum P V) / l with l = sum p (fp32, unrounded).
// Threads, barriers, bounded waits, lazy rescale and the epilogue are those
// of attend.cu.
#include "bsa_device.cuh"
#include "bsa_kernels.h"

namespace bsa {

namespace {

constexpr int kThreads = 384;
constexpr uint32_t kSoftmaxRegs = 232, kControlRegs = 40;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kRing = 12;
constexpr uint32_t kTileBytes = 16384;   // 128 rows x 128 e4m3
constexpr uint32_t kOffQ = 0;            // Q0, Q1
constexpr uint32_t kOffRing = 2 * kTileBytes;
constexpr uint32_t kOffCtl = kOffRing + kRing * kTileBytes;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;
constexpr float kLog2e = 1.4426950408889634074f;
constexpr float kLn2 = 0.69314718055994530942f;
// Lazy rescale threshold (log2 units): p may reach 2^8 (< 448) before O is
// rescaled.
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
  const float* bias;
  const float* q_scale;    // [BH, nb]
  const float* k_scale;    // [BH, nb]
  const float* v_scale;    // [BH, nb]
  const float* ks_scale;   // [BH, ntile]
  const float* vs_scale;   // [BH, ntile]
  const float* v_ref;      // [BH]
  __nv_bfloat16* O;
  float* lse;
  int* dev_status;
  int N, nb, pb, nbv, k_eff, kcap, BH, ntile;
  int prefix_ctas;    // CTAs that take dense-prefix query-block pairs
  float scale_log2;   // log2(e) / sqrt(128)
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtx& wc) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc));
}

// Pair of work items of one CTA: items 2c and 2c+1 of one class (dense-prefix
// query blocks first, then video query blocks, head-major), so both slots
// have the same tile count.
struct Pair {
  int bh[2], qi[2];
  bool act1;
};

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
  for (int s = 0; s < 2; ++s) {
    const int it = min(base + s, count - 1);
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

__global__ void __launch_bounds__(kThreads, 1)
    attend_fp8_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_vt,
                      const __grid_constant__ CUtensorMap tm_ks,
                      const __grid_constant__ CUtensorMap tm_vst, const Args a) {
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

  const Pair pr = pair_of(blockIdx.x, a);
  const bool video = pr.qi[0] >= a.pb;
  const int n_exact = video ? a.pb + a.k_eff : a.nb;
  const bool has_sum = video && (a.k_eff < a.nbv);
  const int u0 = a.pb / kBlock;
  const int T = n_exact + (has_sum ? (a.ntile - u0) : 0);
  const int nslots = pr.act1 ? 2 : 1;

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
    if (warp == kProducerWarp && lane == 0) {
    // ---------------------------------------------------------- producer
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_vt);
      for (int s = 0; s < nslots; ++s) {
        mbar_arrive_expect_tx(&ctl->q_full[s], kTileBytes);
        tma_load_3d(sm + kOffQ + s * kTileBytes, &tm_q, &ctl->q_full[s], 0, pr.qi[s] * kBlock,
                    pr.bh[s]);
      }
      int seq = 0;
      bool ok = true;
      // One operand tile (K or V of slot s, tile t) into the next ring stage.
      // K rows are tokens; V rows are the dimensions of block j (or of
      // summary tile u) at j * 128 (u * 128) in the dimension-major table.
      auto emit = [&](int s, int t, bool is_v) {
        if (!ok) return;
        const int stage = seq % kRing;
        if (seq >= kRing && !mbar_wait(&ctl->empty[stage], ((seq / kRing) - 1) & 1, wc)) {
          ok = false;
          return;
        }
        const CUtensorMap* m;
        int row;
        if (t < n_exact) {
          row = __ldg(a.idx + (static_cast<size_t>(pr.bh[s]) * a.nb + pr.qi[s]) * a.kcap + t) *
                kBlock;
          m = is_v ? &tm_vt : &tm_k;
        } else {
          row = (u0 + t - n_exact) * kBlock;
          m = is_v ? &tm_vst : &tm_ks;
        }
        mbar_arrive_expect_tx(&ctl->full[stage], kTileBytes);
        tma_load_3d(sm + kOffRing + stage * kTileBytes, m, &ctl->full[stage], 0, row, pr.bh[s]);
        ++seq;
      };
      for (int s = 0; s < nslots; ++s) emit(s, 0, false);
      for (int t = 0; t < T && ok; ++t) {
        for (int s = 0; s < nslots; ++s) {
          emit(s, t, true);
          if (t + 1 < T) emit(s, t + 1, false);
        }
      }
      // Drain: every issued load has landed before the CTA exits (immediate
      // on the normal path, where the MMA warp already waited for them).
      for (int s = 0; s < nslots; ++s) mbar_wait(&ctl->q_full[s], 0, wc);
      for (int k = (seq > kRing ? seq - kRing : 0); k < seq; ++k)
        mbar_wait(&ctl->full[k % kRing], (k / kRing) & 1, wc);
    } else if (warp == kMmaWarp && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
      const uint32_t id8 = idesc_e4m3_f32(128, 128);
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
        for (int kk = 0; kk < 4; ++kk) {   // 32 dimensions (bytes) per MMA
          mma_e4m3_ss(tmem + kColS + s * 128, smem_desc_sw128(q_addr + kk * 32, 16, 1024),
                      smem_desc_sw128(k_addr + kk * 32, 16, 1024), id8, kk > 0 ? 1u : 0u);
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
        for (int kk = 0; kk < 4; ++kk) {   // 32 keys per MMA: 8 TMEM columns of P
          mma_e4m3_ts(tmem + kColO + s * 128, tmem + kColS + s * 128 + kk * 8,
                      smem_desc_sw128(v_addr + kk * 32, 16, 1024), id8,
                      (t > 0 || kk > 0) ? 1u : 0u);
        }
        release(stage);
      };
      for (int s = 0; s < nslots && ok; ++s) {
        if (!mbar_wait(&ctl->q_full[s], 0, wc)) ok = false;
      }
      for (int s = 0; s < nslots && ok; ++s) issue_s(s);
      for (int t = 0; t < T && ok; ++t) {
        for (int s = 0; s < nslots && ok; ++s) {
          issue_pv(s, t);
          if (!ok) break;
          if (t + 1 < T) issue_s(s);
          else mma_commit(&ctl->o_final[s]);
        }
      }
      mma_commit(&ctl->fin);
      mbar_wait(&ctl->fin, 0, wc);
    } else if (warp >= 10 && has_sum && warp - 10 < nslots) {
    // ---------------------------------------------------------- bias stager
      // Warp 10 + s stages, for each summary tile v of slot s, the 128 biases
      // in log2 units with -inf where the column is a listed block, a prefix
      // block or past the last block (listed: binary search of the sorted
      // idx row), double buffered against the slot's softmax warps.
      const int s = warp - 10;
      const int32_t* idx_row = a.idx + (static_cast<size_t>(pr.bh[s]) * a.nb + pr.qi[s]) * a.kcap;
      const float* bias_h = a.bias + static_cast<size_t>(pr.bh[s]) * a.nb;
      for (int v = 0; v < T - n_exact; ++v) {
        if (v >= 2 && !warp_wait(&ctl->bias_empty[s][v & 1], ((v >> 1) - 1) & 1, wc)) break;
        float* dst = &ctl->bias_stage[s][v & 1][0];
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          const int c = lane + 32 * q;
          const int j = (u0 + v) * kBlock + c;
          float b = -INFINITY;
          if (j >= a.pb && j < a.nb && !listed(idx_row, a.pb, n_exact, j))
            b = __ldg(bias_h + j) * kLog2e;
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
    const int32_t* idx_row = a.idx + (static_cast<size_t>(bh) * a.nb + qi) * a.kcap;
    const float v_ref = __ldg(a.v_ref + bh);
    const float q_mul = a.scale_log2 * __ldg(a.q_scale + static_cast<size_t>(bh) * a.nb + qi);
    // Per-tile factors (key scale, value scale / v_ref), loaded one tile ahead.
    auto tile_factors = [&](int t, float& k_mul, float& v_mul) {
      if (t < n_exact) {
        const size_t j = static_cast<size_t>(bh) * a.nb + __ldg(idx_row + t);
        k_mul = q_mul * __ldg(a.k_scale + j);
        v_mul = __ldg(a.v_scale + j) / v_ref;
      } else {
        const size_t u = static_cast<size_t>(bh) * a.ntile + u0 + (t - n_exact);
        k_mul = q_mul * __ldg(a.ks_scale + u);
        v_mul = __ldg(a.vs_scale + u) / v_ref;
      }
    };
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = active;
    // Only the last listed block can be the ragged last block (lists are
    // ascending and nb-1 is the largest index): find it once.
    int ragged_t = -1, ragged_cols = kBlock;
    if (active && (a.N % kBlock) != 0 && __ldg(idx_row + n_exact - 1) == a.nb - 1) {
      ragged_t = n_exact - 1;
      ragged_cols = a.N - (a.nb - 1) * kBlock;
    }
    float k_next = 0.f, v_next = 0.f;
    if (active) tile_factors(0, k_next, v_next);
    for (int t = 0; ok && t < T; ++t) {
      const bool exact = t < n_exact;
      const int v = t - n_exact;   // summary tile index when !exact
      const float k_mul = k_next, v_mul = v_next;
      if (t + 1 < T) tile_factors(t + 1, k_next, v_next);
      if (!warp_wait(&ctl->s_full[s], t & 1, wc)) { ok = false; break; }
      tc_fence_after();
      float x[128];
      BSA_TMEM_LD_32F(s_col, x);
      BSA_TMEM_LD_32F(s_col + 32, x + 32);
      BSA_TMEM_LD_32F(s_col + 64, x + 64);
      BSA_TMEM_LD_32F(s_col + 96, x + 96);
      tmem_wait_ld();

      // Exact tiles keep raw code products (the scale is folded into the
      // exponent's FMA; it is > 0 so max commutes with it); summary tiles
      // become logits in log2 units with the staged bias / mask.
      float2 mul = make_float2(k_mul, k_mul);
      if (exact) {
        if (t == ragged_t) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= ragged_cols) x[c] = -INFINITY;
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
      float mp[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mp[k] = x[k];
#pragma unroll
      for (int c = 8; c < 128; ++c) mp[c & 7] = fmaxf(mp[c & 7], x[c]);
      const float mx = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                             fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7]))) * mul.x;
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
      // p = 2^(x * mul - m_new) (row sum in fp32); P = e4m3(p * v_mul), four
      // keys per 32-bit TMEM column.
      const float2 off = make_float2(-m_new, -m_new);
      const float2 vm2 = make_float2(v_mul, v_mul);
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};
      uint32_t pk[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float2 y0 = fma2(make_float2(x[4 * e], x[4 * e + 1]), mul, off);
        const float2 y1 = fma2(make_float2(x[4 * e + 2], x[4 * e + 3]), mul, off);
        const float2 p0 = make_float2(fast_exp2(y0.x), fast_exp2(y0.y));
        const float2 p1 = make_float2(fast_exp2(y1.x), fast_exp2(y1.y));
        acc[(2 * e) & 3] = add2(acc[(2 * e) & 3], p0);
        acc[(2 * e + 1) & 3] = add2(acc[(2 * e + 1) & 3], p1);
        const float2 w0 = mul2(p0, vm2), w1 = mul2(p1, vm2);
        pk[e] = pack_e4m3x4(w0.x, w0.y, w1.x, w1.y);
      }
      BSA_TMEM_ST_32(s_col, pk);
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
      const float inv_l = v_ref / l_run;
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

}  // namespace

cudaError_t launch_attend_fp8(const Shape& s, const AttendMapsFp8& maps, const Fp8Operands& f,
                              const int32_t* idx, const float* bias, void* O, float* lse,
                              cudaStream_t st) {
  constexpr size_t smem = kOffCtl + sizeof(Ctl);
  static std::atomic<bool> attr_set[64];
  cudaError_t e = once_per_device(attr_set, [] {
    return cudaFuncSetAttribute(attend_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                smem);
  });
  if (e != cudaSuccess) return e;
  Args a;
  a.idx = idx;
  a.bias = bias;
  a.q_scale = f.q_scale;
  a.k_scale = f.k_scale;
  a.v_scale = f.v_scale;
  a.ks_scale = f.ks_scale;
  a.vs_scale = f.vs_scale;
  a.v_ref = f.v_ref;
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
  a.ntile = (s.nb + kBlock - 1) / kBlock;
  a.prefix_ctas = (a.BH * s.pb + 1) / 2;
  a.scale_log2 = kLog2e * 0.088388347648318440550f;
  const int grid = a.prefix_ctas + (a.BH * s.nbv + 1) / 2;
  attend_fp8_kernel<<<grid, kThreads, smem, st>>>(maps.q, maps.k, maps.vt, maps.ks, maps.vst, a);
  return cudaGetLastError();
}

}  // namespace bsa
