// Adaptive reblocking of the query/key layout (Spark-Reblock).
//
// Spark-H3 page, section "What Spark-Attn changes", Spark-Reblock bullet: two
// queries are similar when their attention-score patterns over the keys are
// similar (a Mahalanobis cosine induced by the keys' second moment), and a
// hierarchical partitioner splits groups until every leaf holds one block, in
// O(N log N); section "Workflows": keys reuse the query layout (q_reuse_k).
// This library's reading (the pages give no formulas):
//   M = sum_{t >= P} k_t k_t^T;  L L^T = M + 1e-6 * trace(M) / 128 * I;
//   u_t = L^T q_t / |L^T q_t|  (so u . u' is the cosine of the score vectors);
//   a group of n tokens (b = ceil(n/128) >= 2 blocks) is bisected along its
//   principal axis: c = mean u, v = 8 power iterations of the centred scatter
//   sum (u - c)(u - c)^T from (1, ..., 1)/sqrt(128), p = u . v; the
//   floor(b/2)*128 tokens of smallest p (ties to the lower original index) go
//   left.  Leaves are laid out left to right, ascending inside a leaf; the
//   dense prefix rows [0, P) stay in place.
//
// Kernels (all heads of a call at once):
//   gram_kernel<moment>   sum x x^T over the video keys, chunks of 2048 rows:
//                         rows staged through shared memory in the 128-byte
//                         swizzled layout, tcgen05.mma with A = B = rows^T
//                         (MN-major), fp32 accumulator in TMEM; partials per
//                         chunk, reduced in a fixed order by factor_kernel.
//   factor_kernel         Cholesky of M (fp32, one CTA per head); writes
//                         R = L^T as bf16 hi + lo (R ~= hi + lo to ~16 bits).
//   whiten_kernel         Y = Q R^T on tcgen05 (two MMAs per K step: hi, lo),
//                         u = Y / |Y| stored bf16; persistent, one CTA per SM
//                         over consecutive 128-token tiles (R loaded once per
//                         head), TMA ring and two TMEM accumulators.
//   per level (group j of level l found by descending the tree; the groups
//   of a level are ranges of the working order `perm`):
//   gram_kernel<group>    sum u u^T and sum u over a chunk of a group's
//                         rows (gathered through perm); a group that fits in
//                         one chunk finishes its power iteration in the same
//                         CTA, larger groups leave partials for group_kernel.
//   group_reduce_kernel   fixed-order sum of a large group's partials, one
//                         CTA per row of its Gram;
//   group_kernel          then its power iteration.
//   project_kernel        p = u . v per position -> order-preserving key, for
//                         groups of several chunks (a single-chunk group is
//                         projected by its Gram CTA: from the ring, or for more
//                         than 3 tiles from a second pass over its rows).
//   split_kernel          radix select of the floor(b/2)*128-th key (four
//                         8-bit passes over the group's keys, ties broken by
//                         position), then a stable partition of perm
//                         (split_small_kernel: one warp per group where no
//                         group of the level exceeds 1024 keys).
//   permute / unpermute   row gathers of Q, K, V into the new layout and the
//                         scatter of O and lse back.
// Every wait is bounded (globaltimer); on expiry the CTA records
// BSA_ERR_TIMEOUT, drains its MMAs, frees TMEM and returns.
#include "bsa_device.cuh"
#include "bsa_kernels.h"

namespace bsa {

namespace {

constexpr int kChunkTok = 2048;   // rows per Gram chunk (16 tiles)
constexpr int kProjTok = 512;     // positions per projection CTA
constexpr int kPowerIters = 8;
constexpr uint32_t kTile = 32768;          // 128 rows x 128 bf16
constexpr uint32_t kHalf = 16384;          // one 64-column swizzle-atom-wide box

struct Range {
  int start, count;
};

// Group j of level `level`: descend from the root (count <= 128 is a leaf,
// so its descendants do not exist: count 0).
__device__ __forceinline__ Range group_of(int nv, int level, int j) {
  int start = 0, count = nv;
  for (int k = 0; k < level; ++k) {
    if (count <= kBlock) return {0, 0};
    const int m = ((count + kBlock - 1) / kBlock / 2) * kBlock;
    if ((j >> (level - 1 - k)) & 1) {
      start += m;
      count -= m;
    } else {
      count = m;
    }
  }
  return {start, count};
}

// 16-byte chunk c16 (0..15) of row r of a 128 x 128 bf16 tile in the 128-byte
// swizzled layout (two 64-column boxes, rows of 128 bytes, chunk index XOR
// row % 8): the layout the MN-major shared-memory descriptors below expect.
__device__ __forceinline__ uint32_t swz(int r, int c16) {
  return static_cast<uint32_t>((c16 >> 3) * kHalf + r * 128 + ((((c16 & 7) ^ (r & 7))) << 4));
}

// 128 threads, thread i owns row i of G (in g[], overwritten by row i of the
// centred scatter C = G - n c c^T); smem v[128] (16-byte aligned), c[128]
// (mean), red[4].  Writes the unit direction of kPowerIters iterations of C
// from (1, ..., 1)/sqrt(128) to out[i].  A zero step keeps v.
__device__ __forceinline__ void power_iterate(float (&g)[128], float n, float* c, float* v,
                                              float* red, float* out) {
  const int i = threadIdx.x, lane = i & 31, warp = i >> 5;
  const float nci = -n * c[i];
#pragma unroll
  for (int j = 0; j < 128; ++j) g[j] = fmaf(nci, c[j], g[j]);
  v[i] = 0.08838834764831845f;   // 1 / sqrt(128)
  __syncthreads();
  for (int it = 0; it < kPowerIters; ++it) {
    // four independent partial sums (fixed order), v read as broadcast float4s
    float w4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll   // fully: g[] stays in registers
    for (int j4 = 0; j4 < 32; ++j4) {
      const float4 vv = reinterpret_cast<const float4*>(v)[j4];
      w4[0] = fmaf(g[4 * j4], vv.x, w4[0]);
      w4[1] = fmaf(g[4 * j4 + 1], vv.y, w4[1]);
      w4[2] = fmaf(g[4 * j4 + 2], vv.z, w4[2]);
      w4[3] = fmaf(g[4 * j4 + 3], vv.w, w4[3]);
    }
    const float w = (w4[0] + w4[1]) + (w4[2] + w4[3]);
    float s = w * w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) red[warp] = s;
    __syncthreads();
    const float tot = (red[0] + red[1]) + (red[2] + red[3]);
    if (tot > 0.f) v[i] = w / sqrtf(tot);
    __syncthreads();
    if (!(tot > 0.f)) break;
  }
  out[i] = v[i];
}

struct GramArgs {
  const __nv_bfloat16* X;   // moment: K [BH, N, 128]; group: u [BH, nv, 128]
  const int32_t* perm;      // group mode: [BH, N] working order (original indices)
  int N, prefix, nv;
  int level, slots, max_chunks;
  float* part;              // [BH, slots * max_chunks, 128, 128]
  float* psum;              // [BH, slots * max_chunks, 128]  (group mode)
  float* vdir;              // [BH, slots, 128]                (group mode)
  uint32_t* keys;           // [BH, nv] projection keys of small groups (group mode)
  int reduced;              // group_reduce_kernel has summed the partials of this level
  int* dev_status;
};

constexpr int kStages = 3;   // Gram tiles in flight (cp.async ring)
constexpr uint32_t kGramCols = 256;   // TMEM: Gram in columns 0-127, column sums 128-143
// Groups of at most this many rows stay whole in the Gram CTA's ring; the
// CTA forms their projections from it.  Larger single-chunk groups stream
// their rows through the ring once more for the projections (from L2), and
// project_kernel takes only the groups of several chunks.
constexpr int kGramProjRows = kStages * kBlock;

struct GramSmem {
  alignas(1024) uint16_t ones[16 * 64];   // bf16 1.0: B of the column-sum MMAs
  uint64_t done[kStages];
  uint32_t tmem_base;
  int abort_flag;
  alignas(16) float c[128];
  alignas(16) float v[128];
  float red[4];
  int32_t rows[kChunkTok];   // group mode: u row of each position of the chunk
};

template <bool kGroup>
__global__ void __launch_bounds__(128) gram_kernel(const GramArgs a) {
  extern __shared__ __align__(1024) uint8_t sm[];
  GramSmem* ctl = reinterpret_cast<GramSmem*>(sm + kStages * kTile);
  const int tid = threadIdx.x;
  const size_t bh = blockIdx.y;
  int slot = 0, chunk = blockIdx.x, p0, p1;
  Range g{0, a.nv};
  if constexpr (kGroup) {
    slot = blockIdx.x / a.max_chunks;
    chunk = blockIdx.x - slot * a.max_chunks;
    g = group_of(a.nv, a.level, slot);
    if (g.count <= kBlock) return;
  }
  p0 = g.start + chunk * kChunkTok;
  p1 = min(p0 + kChunkTok, g.start + g.count);
  if (p0 >= p1) return;
  const bool single = kGroup && g.count <= kChunkTok;
  if ((smem_u32(sm) & 1023u) != 0) {   // the swizzled layout needs 1024-byte alignment
    if (tid == 0 && a.dev_status) atomicExch(a.dev_status, kErrTimeout);
    return;
  }

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(&ctl->done[i], 1);
    ctl->abort_flag = 0;
    fence_barrier_init();
  }
  if (tid < 32) {
    tmem_alloc(&ctl->tmem_base, kGramCols);
    tmem_relinquish();
  }
  if constexpr (kGroup) {   // the chunk's rows of u, read once; the ones tile
    for (int i = tid; i < p1 - p0; i += 128)
      ctl->rows[i] = __ldg(a.perm + bh * a.N + a.prefix + p0 + i) - a.prefix;
    for (int e = tid; e < 16 * 64; e += 128) ctl->ones[e] = 0x3F80;   // bf16 1.0
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const WaitCtx wc{&ctl->abort_flag, a.dev_status};
  const uint32_t idesc = idesc_bf16_f32_mn(128, 128);
  // column sums: A = rows^T (MN-major) as for the Gram, B = ones (K-major, N = 16)
  constexpr uint32_t idesc_cs = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) |
                                ((16u >> 3) << 17) | ((128u >> 4) << 24);
  const uint32_t ones = smem_u32(ctl->ones);

  auto row_ptr = [&](int pos) -> const __nv_bfloat16* {
    if constexpr (kGroup) {
      return a.X + (bh * a.nv + ctl->rows[pos - p0]) * kDim;
    } else {
      return a.X + (bh * a.N + a.prefix + pos) * kDim;
    }
  };

  const int ntile = (p1 - p0 + kBlock - 1) / kBlock;
  const int c16 = tid & 15;
  // Tiles stream through a ring of kStages buffers with cp.async (16 bytes
  // per copy, rows ps*8 + tid/16), two tiles ahead of the MMA: each thread's
  // copies of a tile form one commit group (empty past the last tile, so the
  // group count stays uniform).  Rows past the chunk are zero-filled.
  auto issue_tile = [&](int it) {
    if (it < ntile) {
      const int base = p0 + it * kBlock;
      const int nrow = min(kBlock, p1 - base);
      uint8_t* buf = sm + (it % kStages) * kTile;
#pragma unroll
      for (int ps = 0; ps < 16; ++ps) {
        const int r = ps * 8 + (tid >> 4);
        const bool valid = r < nrow;
        cp_async16(buf + swz(r, c16),
                   reinterpret_cast<const uint4*>(row_ptr(valid ? base + r : p0)) + c16,
                   valid ? 16u : 0u);
      }
    }
    cp_async_commit();
  };
  issue_tile(0);
  issue_tile(1);
  bool ok = true;
  for (int it = 0; it < ntile && ok; ++it) {
    // buffer (it + 2) % kStages last held tile it - 1: its MMAs must be done
    // and every thread past its column sums before it is refilled
    if (it >= 1) {
      __syncthreads();
      if (!mbar_wait(&ctl->done[(it - 1) % kStages], ((it - 1) / kStages) & 1, wc)) {
        ok = false;
        break;
      }
    }
    issue_tile(it + 2);
    cp_async_wait<2>();   // this thread's copies of tile it have landed
    fence_proxy_async_smem();
    __syncthreads();
    const uint8_t* buf = sm + (it % kStages) * kTile;
    if (tid == 0) {
      tc_fence_after();
      const uint32_t addr = smem_u32(buf);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {   // 16 rows per MMA
        const uint64_t d = smem_desc_sw128(addr + kk * 2048, kHalf, 1024);
        mma_bf16_ss(tmem, d, d, idesc, (it > 0 || kk > 0) ? 1u : 0u);
        if constexpr (kGroup)   // column sums: the same rows times a tile of ones
          mma_bf16_ss(tmem + 128, d, smem_desc_sw128(ones + 32 * (kk & 3), 16, 1024), idesc_cs,
                      (it > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(&ctl->done[it % kStages]);
    }
  }
  cp_async_wait<0>();
  // the last tile's MMAs (all earlier ones complete in order before it)
  const int last = ntile - 1;
  if (ok && !mbar_wait(&ctl->done[last % kStages], (last / kStages) & 1, wc)) ok = false;
  ok = __syncthreads_and(ok);
  tc_fence_after();

  if (ok) {
    const uint32_t lane_base = static_cast<uint32_t>((tid >> 5) * 32) << 16;
    float gr[128];
    BSA_TMEM_LD_32F(tmem + lane_base, gr);
    BSA_TMEM_LD_32F(tmem + lane_base + 32, gr + 32);
    BSA_TMEM_LD_32F(tmem + lane_base + 64, gr + 64);
    BSA_TMEM_LD_32F(tmem + lane_base + 96, gr + 96);
    float colsum = 0.f;
    if constexpr (kGroup) {
      uint32_t cs[8];
      tmem_ld8(tmem + lane_base + 128, cs);
      tmem_wait_ld();
      colsum = __uint_as_float(cs[0]);
    }
    tmem_wait_ld();
    const size_t pidx = static_cast<size_t>(bh) * a.slots * a.max_chunks +
                        static_cast<size_t>(slot) * a.max_chunks + chunk;
    if (single) {
      const float n = static_cast<float>(g.count);
      ctl->c[tid] = colsum / n;
      __syncthreads();
      power_iterate(gr, n, ctl->c, ctl->v, ctl->red,
                    a.vdir + (bh * a.slots + slot) * kDim);
      // p = u . v of every row of the group, summed in project_kernel's
      // order: eight products per 16-byte chunk, then the chunks pairwise as
      // its lane butterfly does.  Thread tid takes row tid of each tile.
      auto project_tile = [&](const uint8_t* buf, int it) {
        const int pos = p0 + it * kBlock + tid;
        if (pos >= p1) return;
        float part[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint4 w = *reinterpret_cast<const uint4*>(buf + swz(tid, c));
          const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&w);
          float sc = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) sc = fmaf(__bfloat162float(h[e]), ctl->v[8 * c + e], sc);
          part[c] = sc;
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1)
#pragma unroll
          for (int c = 0; c < o; ++c) part[c] = part[c] + part[c + o];
        a.keys[bh * a.nv + pos] = orderable_key(part[0]);
      };
      if (g.count <= kGramProjRows) {
        // every tile is still in the ring (tile it in buffer it)
        for (int it = 0; it < ntile; ++it) project_tile(sm + it * kTile, it);
      } else {
        // stream the group's rows through the ring once more (they were just
        // read, so they come from L2)
        issue_tile(0);
        issue_tile(1);
        for (int it = 0; it < ntile; ++it) {
          __syncthreads();   // buffer (it + 2) % kStages (tile it - 1) is done with
          issue_tile(it + 2);
          cp_async_wait<2>();
          __syncthreads();
          project_tile(sm + (it % kStages) * kTile, it);
        }
        cp_async_wait<0>();
      }
    } else {
      float4* dst = reinterpret_cast<float4*>(a.part + (pidx * 128 + tid) * 128);
#pragma unroll
      for (int q = 0; q < 32; ++q)
        dst[q] = make_float4(gr[4 * q], gr[4 * q + 1], gr[4 * q + 2], gr[4 * q + 3]);
      if constexpr (kGroup) a.psum[pidx * 128 + tid] = colsum;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (tid < 32) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kGramCols);
  }
}

// Fixed-order sum of a large group's chunk partials, one CTA per row of its
// Gram (blockIdx.x < 128; the column sums for blockIdx.x == 128), left in the
// group's first partial slot: thread j adds element j of the row chunk by
// chunk, so the sums are those a single thread per row would form.
__global__ void __launch_bounds__(128) group_reduce_kernel(const GramArgs a) {
  const int r = blockIdx.x, slot = blockIdx.y, j = threadIdx.x;
  const size_t bh = blockIdx.z;
  const Range g = group_of(a.nv, a.level, slot);
  if (g.count <= kChunkTok) return;   // leaves and single-chunk groups are done
  const int nch = (g.count + kChunkTok - 1) / kChunkTok;
  const size_t p0 = static_cast<size_t>(bh) * a.slots * a.max_chunks +
                    static_cast<size_t>(slot) * a.max_chunks;
  float acc = 0.f;
  if (r < 128) {
#pragma unroll 4
    for (int ch = 0; ch < nch; ++ch) acc += __ldg(a.part + ((p0 + ch) * 128 + r) * 128 + j);
    a.part[(p0 * 128 + r) * 128 + j] = acc;
  } else {
#pragma unroll 4
    for (int ch = 0; ch < nch; ++ch) acc += __ldg(a.psum + (p0 + ch) * 128 + j);
    a.psum[p0 * 128 + j] = acc;
  }
}

// Power iteration of a group larger than one chunk: on the sums
// group_reduce_kernel left in its first partial slot (a.reduced), or summing
// the chunk partials itself in the same order (groups of a few chunks, where
// a CTA per row would be mostly launch cost).
__global__ void __launch_bounds__(128) group_kernel(const GramArgs a) {
  __shared__ alignas(16) float c[128];
  __shared__ alignas(16) float v[128];
  __shared__ float red[4];
  const int tid = threadIdx.x, slot = blockIdx.x;
  const size_t bh = blockIdx.y;
  const Range g = group_of(a.nv, a.level, slot);
  if (g.count <= kChunkTok) return;   // leaves and single-chunk groups are done
  float gr[128];
#pragma unroll
  for (int j = 0; j < 128; ++j) gr[j] = 0.f;
  float s = 0.f;
  const size_t p0 = static_cast<size_t>(bh) * a.slots * a.max_chunks +
                    static_cast<size_t>(slot) * a.max_chunks;
  const int nch = a.reduced ? 1 : (g.count + kChunkTok - 1) / kChunkTok;
  // chunk by chunk in a fixed order; each chunk's row arrives as 32
  // independent 16-byte loads issued together
  for (int ch = 0; ch < nch; ++ch) {
    const float4* src = reinterpret_cast<const float4*>(a.part + ((p0 + ch) * 128 + tid) * 128);
    float4 x[32];
#pragma unroll
    for (int q = 0; q < 32; ++q) x[q] = __ldg(src + q);
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      gr[4 * q] += x[q].x;
      gr[4 * q + 1] += x[q].y;
      gr[4 * q + 2] += x[q].z;
      gr[4 * q + 3] += x[q].w;
    }
    s += a.psum[(p0 + ch) * 128 + tid];
  }
  const float n = static_cast<float>(g.count);
  c[tid] = s / n;
  __syncthreads();
  power_iterate(gr, n, c, v, red, a.vdir + (bh * a.slots + slot) * kDim);
}

// Fixed-order sum of the key-moment chunk partials: row blockIdx.x of M.
__global__ void __launch_bounds__(128) moment_reduce_kernel(const float* __restrict__ part,
                                                            int nchunk, float* __restrict__ M) {
  const int i = blockIdx.x, j = threadIdx.x;
  const size_t bh = blockIdx.y;
  float s = 0.f;
  for (int ch = 0; ch < nchunk; ++ch) s += part[((bh * nchunk + ch) * 128 + i) * 128 + j];
  M[(bh * 128 + i) * 128 + j] = s;
}

// Cholesky of the key second moment (fp32, in shared memory, lower triangle
// in place) and R = L^T split into bf16 hi + lo.  Right-looking: for each
// column j, the pivot's square root, the column below it scaled, then every
// thread updates its own row of the trailing triangle (independent FMAs).
// fp32 rather than fp64: FP64 runs at about one FMA per SM clock on this
// part (an fp64 version took 0.26 ms for these 350k FMAs per head), and M
// itself arrives as fp32 sums, so a backward-stable fp32 factor (L L^T =
// M + E, |E| <~ 128 * 2^-24 |L| |L^T|) adds an error of the order already in
// M, far below the bf16 rounding of the whitened vectors.  The trace (for
// the ridge) is summed in fp64.
__global__ void __launch_bounds__(128) factor_kernel(const float* __restrict__ Mg,
                                                     __nv_bfloat16* __restrict__ r_hi,
                                                     __nv_bfloat16* __restrict__ r_lo) {
  extern __shared__ float M[];     // [128][129]
  __shared__ double red[128];
  __shared__ float col[128];       // the scaled column j (a separate array: no aliasing)
  const int tid = threadIdx.x;
  const size_t bh = blockIdx.x;
  constexpr int ld = 129;
  // the moment in batches of 16 independent loads per thread
  for (int i0 = 0; i0 < 128; i0 += 16) {
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = __ldg(Mg + (bh * 128 + i0 + i) * 128 + tid);
#pragma unroll
    for (int i = 0; i < 16; ++i) M[(i0 + i) * ld + tid] = x[i];
  }
  __syncthreads();
  red[tid] = M[tid * ld + tid];
  __syncthreads();
  if (tid == 0) {
    double tr = 0.0;
    for (int i = 0; i < 128; ++i) tr += red[i];
    red[0] = 1e-6 * tr / 128.0;
  }
  __syncthreads();
  const float ridge = static_cast<float>(red[0]);
  M[tid * ld + tid] += ridge;
  __syncthreads();
  float* row = M + tid * ld;
  for (int j = 0; j < 128; ++j) {
    // every thread takes the pivot (one broadcast read) and scales its entry
    const float s = M[j * ld + j];
    const float d = sqrtf(s > 0.f ? s : 1e-30f);
    float lij = 0.f;
    if (tid > j) {
      lij = row[j] / d;
      row[j] = lij;
      col[tid] = lij;
    }
    __syncthreads();   // pivot read by all, column j in col[]
    if (tid == j) row[j] = d;
    if (tid > j) {
      // four entries per step: all loads issued before the FMAs and stores
      int k = j + 1;
      for (; k + 3 <= tid; k += 4) {
        const float c0 = col[k], c1 = col[k + 1], c2 = col[k + 2], c3 = col[k + 3];
        const float r0 = row[k], r1 = row[k + 1], r2 = row[k + 2], r3 = row[k + 3];
        row[k] = fmaf(-lij, c0, r0);
        row[k + 1] = fmaf(-lij, c1, r1);
        row[k + 2] = fmaf(-lij, c2, r2);
        row[k + 3] = fmaf(-lij, c3, r3);
      }
      for (; k <= tid; ++k) row[k] = fmaf(-lij, col[k], row[k]);
    }
    __syncthreads();
  }
  // R = L^T: R[i][j] = L[j][i] for j >= i; thread tid writes column j = tid
  for (int i = 0; i < 128; ++i) {
    const float r = tid >= i ? M[tid * ld + i] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(r);
    r_hi[(bh * 128 + i) * 128 + tid] = hi;
    r_lo[(bh * 128 + i) * 128 + tid] = __float2bfloat16_rn(r - __bfloat162float(hi));
  }
}

// AND of `v` over the 128 threads of warps 0-3 (named barrier 1): every one of
// them gets the same answer, so they leave a loop together.
__device__ __forceinline__ bool epi_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, 1, 128, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(v ? 1u : 0u)
      : "memory");
  return r != 0;
}

constexpr int kWhThreads = 192;   // warps 0-3 epilogue (TMEM lane quarters), 4 TMA, 5 MMA
constexpr int kWhStages = 3;      // Q tiles in flight
constexpr uint32_t kWhOffQ = 2 * kTile;                       // after R hi, R lo
constexpr uint32_t kWhOffOut = kWhOffQ + kWhStages * kTile;   // two u tiles for TMA stores
constexpr uint32_t kWhOffCtl = kWhOffOut + 2 * kTile;

struct WhitenSmem {
  uint64_t rfull, rempty;                   // R (hi + lo) of the current head
  uint64_t qfull[kWhStages], qempty[kWhStages];
  uint64_t afull[2], aempty[2];             // two TMEM accumulators
  uint64_t done;                            // every MMA of the CTA complete
  uint32_t tmem_base;
  int abort_flag;
};

// u = Y / |Y|, Y = Q R^T (R ~= hi + lo).  Persistent: CTA c takes the work
// items [c * per, (c + 1) * per) of the (head, 128-token tile) sequence, so
// it loads R once per head it meets; Q tiles stream through a 3-stage TMA
// ring, and the epilogue of one tile (TMEM -> normalise -> store) overlaps
// the MMAs of the next (two accumulators).
__global__ void __launch_bounds__(kWhThreads, 1)
    whiten_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_hi,
                  const __grid_constant__ CUtensorMap tm_lo, const __grid_constant__ CUtensorMap tm_u,
                  int prefix, int nv, int ntile, int total, int per, int* dev_status) {
  extern __shared__ __align__(1024) uint8_t sm[];
  WhitenSmem* ctl = reinterpret_cast<WhitenSmem*>(sm + kWhOffCtl);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int w0 = blockIdx.x * per, w1 = min(total, w0 + per);
  if (w0 >= w1) return;
  const int nw = w1 - w0;
  if (tid == 0) {
    mbar_init(&ctl->rfull, 1);
    mbar_init(&ctl->rempty, 1);
    for (int st = 0; st < kWhStages; ++st) {
      mbar_init(&ctl->qfull[st], 1);
      mbar_init(&ctl->qempty[st], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->afull[b], 1);
      mbar_init(&ctl->aempty[b], 128);
    }
    mbar_init(&ctl->done, 1);
    ctl->abort_flag = ((smem_u32(sm) & 1023u) != 0) ? 1 : 0;
    if (ctl->abort_flag && dev_status) atomicExch(dev_status, kErrTimeout);
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(&ctl->tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const WaitCtx wc{&ctl->abort_flag, dev_status};
  const bool run = ctl->abort_flag == 0;

  if (run && warp == 4) {
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_hi);
      prefetch_tensormap(&tm_lo);
      int cur = -1, nr = 0, issued = 0;
      bool ok = true;
      for (int it = 0; it < nw && ok; ++it) {
        const int w = w0 + it, bh = w / ntile, tile = w - bh * ntile;
        if (bh != cur) {   // R of the new head, once the old head's MMAs are done
          if (nr > 0 && !mbar_wait(&ctl->rempty, (nr - 1) & 1, wc)) { ok = false; break; }
          mbar_arrive_expect_tx(&ctl->rfull, 2 * kTile);
          tma_load_3d(sm, &tm_hi, &ctl->rfull, 0, 0, bh);
          tma_load_3d(sm + kHalf, &tm_hi, &ctl->rfull, 64, 0, bh);
          tma_load_3d(sm + kTile, &tm_lo, &ctl->rfull, 0, 0, bh);
          tma_load_3d(sm + kTile + kHalf, &tm_lo, &ctl->rfull, 64, 0, bh);
          ++nr;
          cur = bh;
        }
        const int st = it % kWhStages;
        if (it >= kWhStages && !mbar_wait(&ctl->qempty[st], ((it / kWhStages) - 1) & 1, wc)) {
          ok = false;
          break;
        }
        uint8_t* dst = sm + kWhOffQ + st * kTile;
        const int row = prefix + tile * kBlock;
        mbar_arrive_expect_tx(&ctl->qfull[st], kTile);
        tma_load_3d(dst, &tm_q, &ctl->qfull[st], 0, row, bh);
        tma_load_3d(dst + kHalf, &tm_q, &ctl->qfull[st], 64, row, bh);
        issued = it + 1;
      }
      // every issued load lands before the CTA moves on
      if (nr > 0) mbar_wait(&ctl->rfull, (nr - 1) & 1, wc);
      for (int k = (issued > kWhStages ? issued - kWhStages : 0); k < issued; ++k)
        mbar_wait(&ctl->qfull[k % kWhStages], (k / kWhStages) & 1, wc);
    }
  } else if (run && warp == 5) {
    if (lane == 0) {
      const uint32_t id = idesc_bf16_f32(128, 128, 0);
      int cur = -1, nr = 0;
      bool ok = true;
      for (int it = 0; it < nw && ok; ++it) {
        const int bh = (w0 + it) / ntile;
        if (bh != cur) {
          if (nr > 0) mma_commit(&ctl->rempty);   // the old head's MMAs release R
          if (!mbar_wait(&ctl->rfull, nr & 1, wc)) { ok = false; break; }
          ++nr;
          cur = bh;
        }
        const int st = it % kWhStages, b = it & 1;
        if (it >= 2 && !mbar_wait(&ctl->aempty[b], ((it >> 1) - 1) & 1, wc)) { ok = false; break; }
        if (!mbar_wait(&ctl->qfull[st], (it / kWhStages) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t q = smem_u32(sm + kWhOffQ + st * kTile);
        for (int part = 0; part < 2; ++part) {
          const uint32_t rr = smem_u32(sm + part * kTile);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
            mma_bf16_ss(tmem + b * 128, smem_desc_sw128(q + off, 16, 1024),
                        smem_desc_sw128(rr + off, 16, 1024), id, (part > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(&ctl->qempty[st]);
        mma_commit(&ctl->afull[b]);
      }
      // TMEM is freed only after every MMA issued here has finished
      mma_commit(&ctl->done);
      mbar_wait(&ctl->done, 0, wc);
    }
  } else if (run) {
    // epilogue: thread tid = TMEM lane = token row of the tile; the tile of
    // u goes to one of two shared buffers in the swizzled layout and leaves
    // by TMA store (rows past nv are not written)
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    for (int it = 0; it < nw; ++it) {
      const int w = w0 + it, bh = w / ntile, tile = w - bh * ntile, b = it & 1;
      // all 128 epilogue threads go on or stop together (named barriers below)
      if (!epi_all(mbar_wait(&ctl->afull[b], (it >> 1) & 1, wc))) break;
      tc_fence_after();
      float y[128];
      BSA_TMEM_LD_32F(tmem + lane_base + b * 128, y);
      BSA_TMEM_LD_32F(tmem + lane_base + b * 128 + 32, y + 32);
      BSA_TMEM_LD_32F(tmem + lane_base + b * 128 + 64, y + 64);
      BSA_TMEM_LD_32F(tmem + lane_base + b * 128 + 96, y + 96);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&ctl->aempty[b]);
      float ss = 0.f;
#pragma unroll
      for (int j = 0; j < 128; ++j) ss = fmaf(y[j], y[j], ss);
      const float inv = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
      // buffer b was last stored from two tiles ago: that store has read it
      if (tid == 0) bulk_wait_group_read<1>();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      uint8_t* out = sm + kWhOffOut + b * kTile;
#pragma unroll
      for (int q = 0; q < 16; ++q)
        *reinterpret_cast<uint4*>(out + swz(tid, q)) =
            make_uint4(pack_bf16x2(y[8 * q] * inv, y[8 * q + 1] * inv),
                       pack_bf16x2(y[8 * q + 2] * inv, y[8 * q + 3] * inv),
                       pack_bf16x2(y[8 * q + 4] * inv, y[8 * q + 5] * inv),
                       pack_bf16x2(y[8 * q + 6] * inv, y[8 * q + 7] * inv));
      fence_proxy_async_smem();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (tid == 0) {
        tma_store_3d(out, &tm_u, 0, tile * kBlock, bh);
        tma_store_3d(out + kHalf, &tm_u, 64, tile * kBlock, bh);
        bulk_commit_group();
      }
    }
    if (tid == 0) bulk_wait_group_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// p = u . v (16 lanes per row, fixed order), stored as an order-preserving key.
__global__ void __launch_bounds__(256) project_kernel(const __nv_bfloat16* __restrict__ u,
                                                      const int32_t* __restrict__ perm,
                                                      const float* __restrict__ vdir, int N,
                                                      int prefix, int nv, int level, int slots,
                                                      int max_pchunks,
                                                      uint32_t* __restrict__ keys) {
  __shared__ float v[128];
  const int tid = threadIdx.x;
  const int slot = blockIdx.x / max_pchunks, chunk = blockIdx.x - slot * max_pchunks;
  const size_t bh = blockIdx.y;
  const Range g = group_of(nv, level, slot);
  if (g.count <= kChunkTok) return;   // leaves; single-chunk groups are done in their Gram CTA
  const int p0 = g.start + chunk * kProjTok, p1 = min(p0 + kProjTok, g.start + g.count);
  if (p0 >= p1) return;
  if (tid < 128) v[tid] = vdir[(bh * slots + slot) * kDim + tid];
  __syncthreads();
  const int c16 = tid & 15;
  float vv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) vv[e] = v[8 * c16 + e];
  // 4 positions per 16-lane group in flight; every half-warp runs the same
  // number of iterations (the shuffles below span the whole warp) and the
  // tail masks the loads instead
  constexpr int kPer = 4;
  for (int base = p0; base < p1; base += 16 * kPer) {
    int orig[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int pos = base + (tid >> 4) + 16 * k;
      orig[k] = pos < p1 ? __ldg(perm + bh * N + prefix + pos) : -1;
    }
    uint4 w[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k)
      w[k] = orig[k] >= 0 ? ld_stream_v4(reinterpret_cast<const uint4*>(
                                             u + (bh * nv + (orig[k] - prefix)) * kDim) + c16)
                          : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&w[k]);
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) s = fmaf(__bfloat162float(h[e]), vv[e], s);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      const int pos = base + (tid >> 4) + 16 * k;
      if (orig[k] >= 0 && c16 == 0) keys[bh * nv + pos] = orderable_key(s);
    }
  }
}

// Exclusive block-wide scan of one int per thread (kSplitThreads threads); returns the
// thread's prefix and writes the block total to *total.
template <int kSplitThreads>
__device__ __forceinline__ int block_scan(int x, int* wsum, int* total) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int w = 0; w < kSplitThreads / 32; ++w) {
      const int t = wsum[w];
      wsum[w] = run;
      run += t;
    }
    *total = run;
  }
  __syncthreads();
  const int res = wsum[warp] + incl - x;
  __syncthreads();
  return res;
}

// Radix select of the m-th smallest key of a group (m = floor(b/2) * 128;
// equal keys count in position order), then the stable partition of perm.
// kSplitThreads: 1024 on levels whose groups are large (the top of the tree,
// few groups), 512 below.
template <int kSplitThreads>
__global__ void __launch_bounds__(kSplitThreads) split_kernel(const uint32_t* __restrict__ keys,
                                                    const int32_t* __restrict__ perm_in,
                                                    int32_t* __restrict__ perm_out, int N,
                                                    int prefix, int nv, int level) {
  __shared__ int hist[256];
  __shared__ int wsum[kSplitThreads / 32];
  __shared__ int sh[4];
  const int tid = threadIdx.x;
  const size_t bh = blockIdx.y;
  const Range g = group_of(nv, level, blockIdx.x);
  if (g.count <= kBlock) return;
  const int m = ((g.count + kBlock - 1) / kBlock / 2) * kBlock;
  const uint32_t* k = keys + bh * nv + g.start;
  uint32_t prefix_bits = 0, mask = 0;
  int want = m;   // rank (1-based) of the wanted key among those matching the prefix
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kSplitThreads) hist[i] = 0;
    __syncthreads();
    for (int i0 = 0; i0 < g.count; i0 += 4 * kSplitThreads) {   // four keys per thread in flight
      uint32_t x[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = i0 + q * kSplitThreads + tid;
        x[q] = i < g.count ? __ldg(k + i) : 0u;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (i0 + q * kSplitThreads + tid < g.count && (x[q] & mask) == prefix_bits)
          atomicAdd(&hist[(x[q] >> shift) & 255u], 1);
    }
    __syncthreads();
    {   // the digit d with (count below d) < want <= (count through d)
      const int h = tid < 256 ? hist[tid] : 0;
      const int below = block_scan<kSplitThreads>(h, wsum, &sh[2]);
      if (tid < 256 && below < want && want <= below + h) {
        sh[0] = tid;
        sh[1] = want - below;
      }
    }
    __syncthreads();
    prefix_bits |= static_cast<uint32_t>(sh[0]) << shift;
    mask |= 255u << shift;
    want = sh[1];
    __syncthreads();
  }
  const uint32_t T = prefix_bits;   // the m-th smallest key
  const int need_eq = want;         // equal keys (in position order) that go left
  int left_run = 0, eq_run = 0;
  const int32_t* pin = perm_in + bh * N + prefix + g.start;
  int32_t* pout = perm_out + bh * N + prefix + g.start;
  uint32_t x_next = tid < g.count ? __ldg(k + tid) : 0xffffffffu;
  for (int base = 0; base < g.count; base += kSplitThreads) {
    const int i = base + tid;
    const bool valid = i < g.count;
    const uint32_t x = x_next;   // loaded one round ahead
    x_next = (i + kSplitThreads < g.count) ? __ldg(k + i + kSplitThreads) : 0xffffffffu;
    const int eq = (valid && x == T) ? 1 : 0;
    int eq_tot;
    const int eq_before = eq_run + block_scan<kSplitThreads>(eq, wsum, &sh[2]);
    eq_tot = sh[2];
    const int left = (valid && (x < T || (eq && eq_before < need_eq))) ? 1 : 0;
    const int l_before = left_run + block_scan<kSplitThreads>(left, wsum, &sh[3]);
    const int l_tot = sh[3];
    if (valid) {
      const int dst = left ? l_before : m + (i - l_before);
      pout[dst] = pin[i];
    }
    left_run += l_tot;
    eq_run += eq_tot;
    __syncthreads();
  }
}

// The same split for a level whose groups hold at most 1024 keys: one warp
// per group, the keys in registers (key of position lane + 32 e in slot e).
// The m-th smallest key T is the (count - m + 1)-th largest, found by a
// bitwise binary search with warp-wide counts; keys below T go left with the
// lowest-position keys equal to T, each side keeping position order.
constexpr int kSplitSmall = 1024;
__global__ void __launch_bounds__(256) split_small_kernel(const uint32_t* __restrict__ keys,
                                                          const int32_t* __restrict__ perm_in,
                                                          int32_t* __restrict__ perm_out, int N,
                                                          int prefix, int nv, int level,
                                                          int slots) {
  const int lane = threadIdx.x & 31;
  const int slot = blockIdx.x * 8 + (threadIdx.x >> 5);
  const size_t bh = blockIdx.y;
  if (slot >= slots) return;
  const Range g = group_of(nv, level, slot);
  if (g.count <= kBlock || g.count > kSplitSmall) return;
  const int m = ((g.count + kBlock - 1) / kBlock / 2) * kBlock;
  const uint32_t* k = keys + bh * nv + g.start;
  uint32_t x[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const int i = lane + 32 * e;
    x[e] = i < g.count ? __ldg(k + i) : 0u;
  }
  // T: the largest value with #{key >= T} >= count - m + 1 (padding is 0 and
  // never counts: every candidate has a bit set)
  const int kth = g.count - m + 1;
  uint32_t T = 0;
  for (int b = 31; b >= 0; --b) {
    const uint32_t cand = T | (1u << b);
    int c = 0;
#pragma unroll
    for (int e = 0; e < 32; ++e) c += (lane + 32 * e < g.count && x[e] >= cand) ? 1 : 0;
    if (__reduce_add_sync(0xffffffffu, c) >= kth) T = cand;
  }
  int lt = 0;
#pragma unroll
  for (int e = 0; e < 32; ++e) lt += (lane + 32 * e < g.count && x[e] < T) ? 1 : 0;
  const int need_eq = m - __reduce_add_sync(0xffffffffu, lt);
  const int32_t* pin = perm_in + bh * N + prefix + g.start;
  int32_t* pout = perm_out + bh * N + prefix + g.start;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int left_run = 0, eq_run = 0;
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    if (32 * e >= g.count) break;
    const int i = lane + 32 * e;
    const bool valid = i < g.count;
    const bool is_eq = valid && x[e] == T;
    const uint32_t eqm = __ballot_sync(0xffffffffu, is_eq);
    const bool left = valid && (x[e] < T || (is_eq && eq_run + __popc(eqm & lt_mask) < need_eq));
    const uint32_t lm = __ballot_sync(0xffffffffu, left);
    const int l_before = left_run + __popc(lm & lt_mask);
    if (valid) pout[left ? l_before : m + (i - l_before)] = __ldg(pin + i);
    left_run += __popc(lm);
    eq_run += __popc(eqm);
  }
}

__global__ void init_perm_kernel(int32_t* __restrict__ perm, int N) {
  const size_t bh = blockIdx.y;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < N; t += gridDim.x * blockDim.x)
    perm[bh * N + t] = t;
}

// Xp[bh][i] = X[bh][perm[bh][i]] for Q, K, V (16 lanes per 256-byte row).
__global__ void __launch_bounds__(256) permute_rows_kernel(const __nv_bfloat16* __restrict__ Q,
                                                           const __nv_bfloat16* __restrict__ K,
                                                           const __nv_bfloat16* __restrict__ V,
                                                           const int32_t* __restrict__ perm,
                                                           int N, __nv_bfloat16* __restrict__ Qp,
                                                           __nv_bfloat16* __restrict__ Kp,
                                                           __nv_bfloat16* __restrict__ Vp) {
  const size_t bh = blockIdx.y;
  const int c16 = threadIdx.x & 15;
  for (int i = blockIdx.x * 16 + (threadIdx.x >> 4); i < N; i += gridDim.x * 16) {
    const size_t src = (bh * N + __ldg(perm + bh * N + i)) * kDim;
    const size_t dst = (bh * N + i) * kDim;
    reinterpret_cast<uint4*>(Qp + dst)[c16] = ld_stream_v4(reinterpret_cast<const uint4*>(Q + src) + c16);
    reinterpret_cast<uint4*>(Kp + dst)[c16] = ld_stream_v4(reinterpret_cast<const uint4*>(K + src) + c16);
    reinterpret_cast<uint4*>(Vp + dst)[c16] = ld_stream_v4(reinterpret_cast<const uint4*>(V + src) + c16);
  }
}

// O[bh][perm[bh][i]] = Op[bh][i] (and lse).
__global__ void __launch_bounds__(256) unpermute_rows_kernel(const __nv_bfloat16* __restrict__ Op,
                                                             const float* __restrict__ lsep,
                                                             const int32_t* __restrict__ perm,
                                                             int N, __nv_bfloat16* __restrict__ O,
                                                             float* __restrict__ lse) {
  const size_t bh = blockIdx.y;
  const int c16 = threadIdx.x & 15;
  for (int i = blockIdx.x * 16 + (threadIdx.x >> 4); i < N; i += gridDim.x * 16) {
    const int t = __ldg(perm + bh * N + i);
    reinterpret_cast<uint4*>(O + (bh * N + t) * kDim)[c16] =
        ld_stream_v4(reinterpret_cast<const uint4*>(Op + (bh * N + i) * kDim) + c16);
    if (lse && c16 == 0) lse[bh * N + t] = lsep[bh * N + i];
  }
}

}  // namespace

// ------------------------------------------------------------------ host side

ReblockPlan reblock_plan(const Shape& s) {
  ReblockPlan p;
  p.nv = s.N - s.prefix;
  p.levels = 0;
  while ((kBlock << p.levels) < p.nv) ++p.levels;   // ceil(log2(ceil(nv / 128)))
  p.moment_chunks = (p.nv + kChunkTok - 1) / kChunkTok;
  p.max_partials = 1;
  int largest = p.nv;   // the rightmost group is the largest of its level
  for (int l = 0; l < p.levels; ++l) {
    const int chunks = (largest + kChunkTok - 1) / kChunkTok;
    p.max_chunks[l] = chunks;
    // the rightmost group is the largest: none left for project_kernel when
    // it fits in one Gram chunk
    p.max_pchunks[l] = largest > kChunkTok ? (largest + kProjTok - 1) / kProjTok : 0;
    p.largest[l] = largest;
    const long long parts = (chunks > 1) ? (static_cast<long long>(1) << l) * chunks : 1;
    if (parts > p.max_partials) p.max_partials = static_cast<int>(parts);
    const int m = ((largest + kBlock - 1) / kBlock / 2) * kBlock;
    largest -= m;
  }
  if (p.moment_chunks > p.max_partials) p.max_partials = p.moment_chunks;
  return p;
}

cudaError_t launch_reblock(const Shape& s, const ReblockPlan& plan, const void* Q, const void* K,
                           const ReblockMaps& maps, const ReblockBuffers& w, int32_t* perm_out,
                           cudaStream_t st) {
  const int BH = s.B * s.H;
  const int nv = plan.nv;
  // Gram kernels: three 32 KB tiles + control; factor: 128 x 129 floats.
  const size_t gram_smem = kStages * kTile + sizeof(GramSmem) + 1024;
  const size_t whiten_smem = kWhOffCtl + sizeof(WhitenSmem) + 1024;
  const size_t factor_smem = 128 * 129 * sizeof(float);
  static std::atomic<bool> attr[64];
  cudaError_t ea = once_per_device(attr, [&] {
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(gram_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  gram_smem)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(gram_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  gram_smem)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(whiten_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  whiten_smem)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(factor_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  factor_smem)) != cudaSuccess)
      return e;
    return cudaSuccess;
  });
  if (ea != cudaSuccess) return ea;
  int32_t* pa = perm_out;
  int32_t* pb = w.perm_tmp;
  init_perm_kernel<<<dim3(64, BH), 256, 0, st>>>(pa, s.N);
  if (plan.levels == 0) return cudaGetLastError();

  GramArgs ga{};
  ga.N = s.N;
  ga.prefix = s.prefix;
  ga.nv = nv;
  ga.part = w.part;
  ga.psum = w.psum;
  ga.vdir = w.vdir;
  ga.keys = w.keys;
  ga.dev_status = s.dev_status;
  // 1. key second moment (chunk partials), 2. factor, 3. whiten
  ga.X = static_cast<const __nv_bfloat16*>(K);
  ga.perm = nullptr;
  ga.level = 0;
  ga.slots = 1;
  ga.max_chunks = plan.moment_chunks;
  gram_kernel<false><<<dim3(plan.moment_chunks, BH), 128, gram_smem, st>>>(ga);
  moment_reduce_kernel<<<dim3(128, BH), 128, 0, st>>>(w.part, plan.moment_chunks, w.moment);
  factor_kernel<<<BH, 128, factor_smem, st>>>(w.moment, w.r_hi, w.r_lo);
  {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int ntile = (nv + kBlock - 1) / kBlock;
    const int total = BH * ntile;
    const int ctas = total < sms ? total : sms;
    const int per = (total + ctas - 1) / ctas;
    whiten_kernel<<<(total + per - 1) / per, kWhThreads, whiten_smem, st>>>(
        maps.q, maps.r_hi, maps.r_lo, maps.u, s.prefix, nv, ntile, total, per, s.dev_status);
  }
  (void)Q;
  // 4. levels
  ga.X = w.u;
  for (int l = 0; l < plan.levels; ++l) {
    const int slots = 1 << l;
    cudaError_t e = cudaMemcpyAsync(pb, pa, static_cast<size_t>(BH) * s.N * sizeof(int32_t),
                                    cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return e;
    ga.perm = pa;
    ga.level = l;
    ga.slots = slots;
    ga.max_chunks = plan.max_chunks[l];
    gram_kernel<true><<<dim3(slots * plan.max_chunks[l], BH), 128, gram_smem, st>>>(ga);
    if (plan.max_chunks[l] > 1) {
      // a CTA per Gram row for groups of 4 or more chunks (768p-5s level 0,
      // 18 chunks: 67 -> 28 us); a CTA per group below that
      ga.reduced = plan.max_chunks[l] >= 4 ? 1 : 0;
      if (ga.reduced) group_reduce_kernel<<<dim3(129, slots, BH), 128, 0, st>>>(ga);
      group_kernel<<<dim3(slots, BH), 128, 0, st>>>(ga);
    }
    if (plan.max_pchunks[l] > 0)
      project_kernel<<<dim3(slots * plan.max_pchunks[l], BH), 256, 0, st>>>(
          w.u, pa, w.vdir, s.N, s.prefix, nv, l, slots, plan.max_pchunks[l], w.keys);
    if (plan.largest[l] <= kSplitSmall)
      split_small_kernel<<<dim3((slots + 7) / 8, BH), 256, 0, st>>>(w.keys, pa, pb, s.N,
                                                                    s.prefix, nv, l, slots);
    else
      if (plan.largest[l] > 8192)   // measured: 106 -> 68 us at level 0 of 768p-5s
        split_kernel<1024><<<dim3(slots, BH), 1024, 0, st>>>(w.keys, pa, pb, s.N, s.prefix, nv, l);
      else
        split_kernel<512><<<dim3(slots, BH), 512, 0, st>>>(w.keys, pa, pb, s.N, s.prefix, nv, l);
    int32_t* t = pa;
    pa = pb;
    pb = t;
  }
  if (pa != perm_out) {
    cudaError_t e = cudaMemcpyAsync(perm_out, pa, static_cast<size_t>(BH) * s.N * sizeof(int32_t),
                                    cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

cudaError_t launch_permute_rows(const Shape& s, const void* Q, const void* K, const void* V,
                                const int32_t* perm, void* Qp, void* Kp, void* Vp,
                                cudaStream_t st) {
  const int BH = s.B * s.H;
  const int blocks = (s.N + 15) / 16 < 1024 ? (s.N + 15) / 16 : 1024;
  permute_rows_kernel<<<dim3(blocks, BH), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K),
      static_cast<const __nv_bfloat16*>(V), perm, s.N, static_cast<__nv_bfloat16*>(Qp),
      static_cast<__nv_bfloat16*>(Kp), static_cast<__nv_bfloat16*>(Vp));
  return cudaGetLastError();
}

cudaError_t launch_unpermute_rows(const Shape& s, const void* Op, const float* lsep,
                                  const int32_t* perm, void* O, float* lse, cudaStream_t st) {
  const int BH = s.B * s.H;
  const int blocks = (s.N + 15) / 16 < 1024 ? (s.N + 15) / 16 : 1024;
  unpermute_rows_kernel<<<dim3(blocks, BH), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(Op), lsep, perm, s.N, static_cast<__nv_bfloat16*>(O),
      lse);
  return cudaGetLastError();
}

}  // namespace bsa
