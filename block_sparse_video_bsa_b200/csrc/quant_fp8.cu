// FP8 (e4m3) operands of the attention kernel: per-group quantisation.
//
// The pages name a quantised sparse kernel ("H3 Sparse Attention", comfy.icu
// WAS node, section "What it actually does": the sparse layers compute in
// INT8 inside the kernel).  Format, granularity and rounding are this
// library's choice: e4m3, one scale per 128-row group (a 128-token block of
// Q, K or V; a 128-row tile of the summary tables), codes
// rn_satfinite_e4m3(x * fp32(448 / amax)) and dequantisation scale
// fp32(amax / 448); an all-zero group has ratio and scale 1.
//
// One CTA of 256 threads per (group, head): 16 threads cover one 256-byte
// bf16 row with 16-byte loads, 16 rows per pass, 8 passes; every element is
// read once.  Codes are written row-major ([rows, 128], the layout of the
// input) or, for the value side, dimension-major per group ([128 dims, 128
// rows], zero past the last row) through a shared-memory transpose, so that
// the PV MMA reads V K-major.
#include "bsa_device.cuh"
#include "bsa_kernels.h"

namespace bsa {

namespace {

constexpr int kThreads = 256;

// Byte (r, c) of the 128 x 128-byte transpose tile: 16-byte chunks of a row
// are XOR-swizzled by r / 16, so the column reads of the transpose (16 rows
// r0..r0+15 of 4 adjacent columns per 4 lanes, 8 row groups per warp) touch 8
// different banks.
__device__ __forceinline__ int tswz(int r, int c) {
  return r * 128 + ((((c >> 4) ^ (r >> 4)) & 7) << 4) + (c & 15);
}

template <bool kTranspose>
__global__ void __launch_bounds__(kThreads) quant_kernel(const __nv_bfloat16* __restrict__ X,
                                                         int rows, int groups,
                                                         uint8_t* __restrict__ codes,
                                                         float* __restrict__ scale) {
  __shared__ float red[kThreads / 32];
  __shared__ __align__(16) uint8_t tile[kTranspose ? 128 * 128 : 16];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = blockIdx.x;
  const size_t bh = blockIdx.y;
  const int r0 = g * kBlock;
  const int nrows = min(kBlock, rows - r0);
  const int c8 = tid & 15;        // 8-element column chunk
  const int rsub = tid >> 4;      // row within a pass

  float x[8][8];
  float amax = 0.f;
#pragma unroll
  for (int ps = 0; ps < 8; ++ps) {
    const int r = ps * 16 + rsub;
    uint4 w = make_uint4(0, 0, 0, 0);
    if (r < nrows)
      w = ld_stream_v4(reinterpret_cast<const uint4*>(X + ((bh * rows + r0 + r) * kDim)) + c8);
    const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&w);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      x[ps][e] = __bfloat162float(h[e]);
      amax = fmaxf(amax, fabsf(x[ps][e]));
    }
  }
  // |x| >= 0, so the float's bits order like unsigned integers.
  uint32_t m = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
  if (lane == 0) red[warp] = __uint_as_float(m);
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) amax = fmaxf(amax, red[w]);
  const float ratio = amax > 0.f ? __fdiv_rn(448.f, amax) : 1.f;
  if (tid == 0) scale[bh * groups + g] = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;

#pragma unroll
  for (int ps = 0; ps < 8; ++ps) {
    const int r = ps * 16 + rsub;
    uint32_t w0 = pack_e4m3x4(__fmul_rn(x[ps][0], ratio), __fmul_rn(x[ps][1], ratio),
                              __fmul_rn(x[ps][2], ratio), __fmul_rn(x[ps][3], ratio));
    uint32_t w1 = pack_e4m3x4(__fmul_rn(x[ps][4], ratio), __fmul_rn(x[ps][5], ratio),
                              __fmul_rn(x[ps][6], ratio), __fmul_rn(x[ps][7], ratio));
    if (r >= nrows) w0 = w1 = 0u;
    if constexpr (kTranspose) {
      *reinterpret_cast<uint2*>(tile + tswz(r, 8 * c8)) = make_uint2(w0, w1);
    } else if (r < nrows) {
      *reinterpret_cast<uint2*>(codes + (bh * rows + r0 + r) * kDim + 8 * c8) = make_uint2(w0, w1);
    }
  }
  if constexpr (kTranspose) {
    __syncthreads();
    // Output [128 dims][128 rows] of this group: thread -> (dim, 16-row chunk).
    uint8_t* out = codes + (bh * groups + g) * static_cast<size_t>(kBlock * kDim);
    for (int it = tid; it < kDim * (kBlock / 16); it += kThreads) {
      const int dim = it >> 3, rc = it & 7;
      uint32_t w[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t v = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b)
          v |= static_cast<uint32_t>(tile[tswz(rc * 16 + q * 4 + b, dim)]) << (8 * b);
        w[q] = v;
      }
      *reinterpret_cast<uint4*>(out + dim * kBlock + rc * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// Largest value-side scale of each head (blocks of V and tiles of v~): the
// attention kernel scales its e4m3 numerators by scale / v_ref <= 1.
__global__ void v_ref_kernel(const float* __restrict__ v_scale, const float* __restrict__ vs_scale,
                             int nb, int ntile, float* __restrict__ v_ref) {
  const size_t bh = blockIdx.x;
  float m = 0.f;
  for (int j = threadIdx.x; j < nb; j += 32) m = fmaxf(m, v_scale[bh * nb + j]);
  for (int j = threadIdx.x; j < ntile; j += 32) m = fmaxf(m, vs_scale[bh * ntile + j]);
  m = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(m)));
  if (threadIdx.x == 0) v_ref[bh] = m;
}

}  // namespace

cudaError_t launch_quantize_fp8(const Shape& s, const void* Q, const void* K, const void* V,
                                const void* ksum, const void* vsum, const Fp8Operands& f,
                                cudaStream_t st) {
  const int BH = s.B * s.H;
  const int ntile = (s.nb + kBlock - 1) / kBlock;
  const dim3 gN(s.nb, BH), gS(ntile, BH);
  quant_kernel<false><<<gN, kThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(Q), s.N, s.nb,
                                               static_cast<uint8_t*>(f.q8), f.q_scale);
  quant_kernel<false><<<gN, kThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(K), s.N, s.nb,
                                               static_cast<uint8_t*>(f.k8), f.k_scale);
  quant_kernel<true><<<gN, kThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(V), s.N, s.nb,
                                              static_cast<uint8_t*>(f.vt8), f.v_scale);
  quant_kernel<false><<<gS, kThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(ksum), s.nb, ntile,
                                               static_cast<uint8_t*>(f.ks8), f.ks_scale);
  quant_kernel<true><<<gS, kThreads, 0, st>>>(static_cast<const __nv_bfloat16*>(vsum), s.nb, ntile,
                                              static_cast<uint8_t*>(f.vst8), f.vs_scale);
  v_ref_kernel<<<BH, 32, 0, st>>>(f.v_scale, f.vs_scale, s.nb, ntile, f.v_ref);
  return cudaGetLastError();
}

}  // namespace bsa
