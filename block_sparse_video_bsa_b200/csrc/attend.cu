// Exact branch + compressed branch of block-sparse attention on tcgen05.
//
// "Block sparse attention splits a video attention pass into two branches:
// an exact branch that computes the top-ranked key/value blocks in full, and
// a compressed branch that covers everything else" (Spark-H3 page, section
// "What Spark-Attn changes").  For one query block (128 rows) this kernel
// streams, as 128-key tiles:
//   * the listed key blocks idx[0..cnt) (exact branch; the ragged last block
//     is masked by column), then
//   * the summary rows k~_j / v~_j of all video blocks, 128 per tile, with
//     logit + bias_j, and the listed / prefix / out-of-range columns masked
//     (compressed branch),
// through one online softmax, so both branches share the running max and sum.
//
// One CTA per query block, 256 threads in four roles:
//   warp 0      TMA producer: Q once, then K / V tiles gathered by block index
//               (3-D tensor maps [B*H, rows, 128], 128-byte swizzle; rows past
//               the end of a head are zero-filled by the TMA unit).
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer:
//               S[t&1] = Q K_t^T  (M=N=128, K=128, both K-major), then
//               O     += P_t V_t  (A = P from shared memory, B = V MN-major).
//   warps 4-7   softmax: one thread per query row (TMEM lane = row), fp32
//               online softmax in base 2 with lazy rescaling of O (only when
//               the running max grows by more than 2^8), P written as bf16
//               into the swizzled shared-memory operand layout; epilogue
//               O / l -> bf16 and lse.
// TMEM: S0 cols [0,128), S1 [128,256), O [256,384) of a 512-column block.
// Shared memory: Q 32 KB, K 2 x 32 KB, V 2 x 32 KB, P 32 KB, barriers, and a
// bitmap of the listed blocks for masking the summary columns.
// Every mbarrier wait is bounded (bsa_device.cuh); on expiry the CTA records
// BSA_ERR_TIMEOUT, drains what it issued, frees TMEM and returns.
#include "bsa_device.cuh"
#include "bsa_kernels.h"

namespace bsa {

namespace {

constexpr int kThreads = 256;
constexpr uint32_t kTileBytes = 32768;   // 128 x 128 bf16
constexpr uint32_t kSubBytes = 16384;    // 128 rows x 64 bf16 (one 128-byte swizzle atom wide)
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kTileBytes;       // 2 stages
constexpr uint32_t kOffV = kOffK + 2 * kTileBytes;   // 2 stages
constexpr uint32_t kOffP = kOffV + 2 * kTileBytes;
constexpr uint32_t kOffCtl = kOffP + kTileBytes;     // 196608
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;
constexpr float kLog2e = 1.4426950408889634074f;
constexpr float kLn2 = 0.69314718055994530942f;
// Lazy rescale threshold (log2 units): p may reach 2^8 before O is rescaled.
constexpr float kRescaleThreshold = 8.0f;

struct Ctl {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full, pv_done, fin;
  uint64_t bias_full[2];
  uint32_t tmem_base;
  int abort_flag;
  int skip;
  alignas(16) float bias_stage[2][128];   // masked bias of the current summary tile
  uint32_t bitmap[1];   // ceil(nb / 32) words follow
};

struct Args {
  const int32_t* idx;
  const int32_t* cnt;
  const float* bias;
  __nv_bfloat16* O;
  float* lse;
  int* dev_status;
  int N, nb, pb, nbv, k_eff, kcap, BH;
  float scale_log2;   // log2(e) / sqrt(128)
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtx& wc) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc));
}

__global__ void __launch_bounds__(kThreads, 1)
    attend_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_ks,
                  const __grid_constant__ CUtensorMap tm_vs, const Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  Ctl* ctl = reinterpret_cast<Ctl*>(sm + kOffCtl);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // A CTA that starts after another one recorded an expired wait does nothing
  // (decided by one thread so that the whole CTA takes the same branch).
  if (tid == 0)
    ctl->skip = (a.dev_status && *reinterpret_cast<volatile int*>(a.dev_status) != 0) ? 1 : 0;
  __syncthreads();
  if (ctl->skip) return;

  // Work item: dense-prefix query blocks first (they are the long ones),
  // then video query blocks, head-major so concurrent CTAs share K/V in L2.
  int item = blockIdx.x, bh, qi;
  const int n_prefix_items = a.BH * a.pb;
  if (item < n_prefix_items) {
    bh = item / a.pb;
    qi = item - bh * a.pb;
  } else {
    item -= n_prefix_items;
    bh = item / a.nbv;
    qi = a.pb + (item - bh * a.nbv);
  }
  const int32_t* idx_row = a.idx + (static_cast<size_t>(bh) * a.nb + qi) * a.kcap;
  const int n_exact = __ldg(a.cnt + static_cast<size_t>(bh) * a.nb + qi);
  const bool has_sum = (qi >= a.pb) && (a.k_eff < a.nbv);
  const int u0 = a.pb / kBlock;
  const int n_tiles = n_exact + (has_sum ? ((a.nb + kBlock - 1) / kBlock - u0) : 0);
  const int nbw = (a.nb + 31) / 32;

  if (tid == 0) {
    mbar_init(&ctl->q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ctl->k_full[s], 1);
      mbar_init(&ctl->k_empty[s], 1);
      mbar_init(&ctl->v_full[s], 1);
      mbar_init(&ctl->v_empty[s], 1);
      mbar_init(&ctl->s_full[s], 1);
      mbar_init(&ctl->s_free[s], 128);
    }
    mbar_init(&ctl->p_full, 128);
    mbar_init(&ctl->pv_done, 1);
    mbar_init(&ctl->fin, 1);
    mbar_init(&ctl->bias_full[0], 128);
    mbar_init(&ctl->bias_full[1], 128);
    ctl->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (has_sum) {
    for (int w = tid; w < nbw; w += kThreads) ctl->bitmap[w] = 0u;
    __syncthreads();
    for (int t = a.pb + tid; t < n_exact; t += kThreads) {
      const int j = __ldg(idx_row + t);
      atomicOr(&ctl->bitmap[j >> 5], 1u << (j & 31));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const WaitCtx wc{&ctl->abort_flag, a.dev_status};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_tiles > 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      mbar_arrive_expect_tx(&ctl->q_full, kTileBytes);
      tma_load_3d(sm + kOffQ, &tm_q, &ctl->q_full, 0, qi * kBlock, bh);
      tma_load_3d(sm + kOffQ + kSubBytes, &tm_q, &ctl->q_full, 64, qi * kBlock, bh);
      int k_last[2] = {-1, -1}, v_last[2] = {-1, -1};
      for (int t = 0; t < n_tiles; ++t) {
        const int st = t & 1;
        const CUtensorMap *mk, *mv;
        int row;
        if (t < n_exact) {
          row = __ldg(idx_row + t) * kBlock;
          mk = &tm_k;
          mv = &tm_v;
        } else {
          row = (u0 + t - n_exact) * kBlock;
          mk = &tm_ks;
          mv = &tm_vs;
        }
        if (t >= 2 && !mbar_wait(&ctl->k_empty[st], ((t >> 1) - 1) & 1, wc)) break;
        uint8_t* kd = sm + kOffK + st * kTileBytes;
        mbar_arrive_expect_tx(&ctl->k_full[st], kTileBytes);
        tma_load_3d(kd, mk, &ctl->k_full[st], 0, row, bh);
        tma_load_3d(kd + kSubBytes, mk, &ctl->k_full[st], 64, row, bh);
        k_last[st] = t;
        if (t >= 2 && !mbar_wait(&ctl->v_empty[st], ((t >> 1) - 1) & 1, wc)) break;
        uint8_t* vd = sm + kOffV + st * kTileBytes;
        mbar_arrive_expect_tx(&ctl->v_full[st], kTileBytes);
        tma_load_3d(vd, mv, &ctl->v_full[st], 0, row, bh);
        tma_load_3d(vd + kSubBytes, mv, &ctl->v_full[st], 64, row, bh);
        v_last[st] = t;
      }
      // Drain: every load this thread issued has landed before the CTA exits
      // (immediate on the normal path, where the consumer already waited).
      mbar_wait(&ctl->q_full, 0, wc);
      for (int s = 0; s < 2; ++s) {
        if (k_last[s] >= 0) mbar_wait(&ctl->k_full[s], (k_last[s] >> 1) & 1, wc);
        if (v_last[s] >= 0) mbar_wait(&ctl->v_full[s], (v_last[s] >> 1) & 1, wc);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_tiles > 0) {
      const uint32_t id_s = idesc_bf16_f32(128, 128, 0);
      const uint32_t id_pv = idesc_bf16_f32(128, 128, 1);
      const uint32_t q_addr = smem_u32(sm + kOffQ);
      const uint32_t p_addr = smem_u32(sm + kOffP);
      bool ok = mbar_wait(&ctl->q_full, 0, wc);
      for (int t = 0; ok && t <= n_tiles; ++t) {
        if (t < n_tiles) {
          const int st = t & 1;
          if (!mbar_wait(&ctl->k_full[st], (t >> 1) & 1, wc)) break;
          if (t >= 2 && !mbar_wait(&ctl->s_free[st], ((t >> 1) - 1) & 1, wc)) break;
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sm + kOffK + st * kTileBytes);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kSubBytes + (kk & 3) * 32;
            mma_bf16_ss(tmem + kColS + st * 128, smem_desc_sw128(q_addr + off, 16, 1024),
                        smem_desc_sw128(k_addr + off, 16, 1024), id_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(&ctl->s_full[st]);
          mma_commit(&ctl->k_empty[st]);
        }
        if (t >= 1) {
          const int tp = t - 1, st = tp & 1;
          if (!mbar_wait(&ctl->v_full[st], (tp >> 1) & 1, wc)) break;
          if (!mbar_wait(&ctl->p_full, tp & 1, wc)) break;
          tc_fence_after();
          const uint32_t v_addr = smem_u32(sm + kOffV + st * kTileBytes);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            mma_bf16_ss(tmem + kColO,
                        smem_desc_sw128(p_addr + (kk >> 2) * kSubBytes + (kk & 3) * 32, 16, 1024),
                        smem_desc_sw128(v_addr + kk * 2048, kSubBytes, 1024), id_pv,
                        (tp > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&ctl->pv_done);
          mma_commit(&ctl->v_empty[st]);
        }
      }
      mma_commit(&ctl->fin);
      mbar_wait(&ctl->fin, 0, wc);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int r = tid - 128;                       // query row within the block
    const uint32_t lane_base = static_cast<uint32_t>((warp - 4) * 32) << 16;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = n_tiles > 0;
    uint8_t* prow = sm + kOffP + r * 128;
    const float* bias_h = a.bias + static_cast<size_t>(bh) * a.nb;
    float* ctl_bias = &ctl->bias_stage[0][0];
    for (int t = 0; ok && t < n_tiles; ++t) {
      const int sb = t & 1;
      if (t >= n_exact) {
        // Stage summary tile v's bias in log2 units, -inf where the column is
        // a listed block, a prefix block or past the last block.  Buffer v&1
        // is free again: every reader of its previous use (tile t-2) finished
        // that tile before PV(t-2) could run, and this thread waited for
        // PV(t-2) in tile t-1.
        const int v = t - n_exact;
        const int j = (u0 + v) * kBlock + r;
        float b = -INFINITY;
        if (j >= a.pb && j < a.nb && !((ctl->bitmap[j >> 5] >> (j & 31)) & 1u))
          b = __ldg(bias_h + j) * kLog2e;
        ctl_bias[(v & 1) * 128 + r] = b;
        mbar_arrive(&ctl->bias_full[v & 1]);
        if (!warp_wait(&ctl->bias_full[v & 1], (v >> 1) & 1, wc)) { ok = false; break; }
      }
      if (!warp_wait(&ctl->s_full[sb], (t >> 1) & 1, wc)) { ok = false; break; }
      tc_fence_after();
      float x[128];
      const uint32_t sa = tmem + lane_base + kColS + sb * 128;
      BSA_TMEM_LD_32F(sa, x);
      BSA_TMEM_LD_32F(sa + 32, x + 32);
      BSA_TMEM_LD_32F(sa + 64, x + 64);
      BSA_TMEM_LD_32F(sa + 96, x + 96);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&ctl->s_free[sb]);

      if (t < n_exact) {
        const int j = __ldg(idx_row + t);
        const int ncols = min(kBlock, a.N - j * kBlock);
#pragma unroll
        for (int c = 0; c < 128; ++c) x[c] = (c < ncols) ? x[c] * a.scale_log2 : -INFINITY;
      } else {
        const float4* bb4 = reinterpret_cast<const float4*>(ctl_bias + ((t - n_exact) & 1) * 128);
#pragma unroll
        for (int c4 = 0; c4 < 32; ++c4) {
          const float4 b = bb4[c4];
          x[4 * c4 + 0] = fmaf(x[4 * c4 + 0], a.scale_log2, b.x);
          x[4 * c4 + 1] = fmaf(x[4 * c4 + 1], a.scale_log2, b.y);
          x[4 * c4 + 2] = fmaf(x[4 * c4 + 2], a.scale_log2, b.z);
          x[4 * c4 + 3] = fmaf(x[4 * c4 + 3], a.scale_log2, b.w);
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) mx = fmaxf(mx, x[c]);
      const bool need = mx > m_run + kRescaleThreshold;
      const float m_new = need ? mx : m_run;
      const float alpha = need ? fast_exp2(m_run - m_new) : 1.0f;
      if (t > 0) {
        // PV(t-1) done: the P buffer is free and O is stable
        if (!warp_wait(&ctl->pv_done, (t - 1) & 1, wc)) { ok = false; break; }
        tc_fence_after();
      }
      float rs = 0.f;
#pragma unroll
      for (int c8 = 0; c8 < 16; ++c8) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p0 = fast_exp2(x[c8 * 8 + 2 * e] - m_new);
          const float p1 = fast_exp2(x[c8 * 8 + 2 * e + 1] - m_new);
          rs += p0 + p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        const int sub = c8 >> 3, cc = c8 & 7;
        *reinterpret_cast<uint4*>(prow + sub * kSubBytes + ((cc ^ (r & 7)) << 4)) =
            make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      if (t > 0 && __any_sync(0xffffffffu, need)) {
        const uint32_t oa = tmem + lane_base + kColO;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float o[32];
          BSA_TMEM_LD_32F(oa + q * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= alpha;
          BSA_TMEM_ST_32(oa + q * 32, reinterpret_cast<uint32_t*>(o));
        }
        tmem_wait_st();
      }
      m_run = m_new;
      l_run = l_run * alpha + rs;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&ctl->p_full);
    }
    // ---------------------------------------------------------- epilogue
    if (ok && warp_wait(&ctl->pv_done, (n_tiles - 1) & 1, wc)) {
      tc_fence_after();
      const int qrow = qi * kBlock + r;
      const bool live = qrow < a.N;
      const float inv_l = 1.f / l_run;
      uint4* orow = reinterpret_cast<uint4*>(a.O + (static_cast<size_t>(bh) * a.N + qrow) * kDim);
      const uint32_t oa = tmem + lane_base + kColO;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float o[32];
        BSA_TMEM_LD_32F(oa + q * 32, o);
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
  if (warp == 1) {
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

static size_t attend_smem_bytes(int nb) {
  // bitmap words plus 4 spare words, so no guarded read can leave the allocation
  return 1024 + kOffCtl + sizeof(Ctl) + sizeof(uint32_t) * ((nb + 31) / 32 + 4);
}

cudaError_t launch_attend(const Shape& s, const AttendMaps& maps, const int32_t* idx,
                          const int32_t* cnt, const float* bias, void* O, float* lse,
                          cudaStream_t st) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         227 * 1024);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  Args a;
  a.idx = idx;
  a.cnt = cnt;
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
  a.scale_log2 = kLog2e * 0.088388347648318440550f;
  const int grid = a.BH * s.nb;
  attend_kernel<<<grid, kThreads, attend_smem_bytes(s.nb), st>>>(maps.q, maps.k, maps.v, maps.ks,
                                                                 maps.vs, a);
  return cudaGetLastError();
}

cudaError_t launch_expired_wait(int32_t* dev_status, uint64_t timeout_ns, cudaStream_t st) {
  expired_wait_kernel<<<1, 32, 0, st>>>(dev_status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace bsa
