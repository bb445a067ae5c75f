// C ABI of libbsa.so (declared in include/bsa.h): argument checks, TMA
// tensor-map construction and the launches of the four stages.  No memory is
// allocated here and no state is kept between calls except per-device
// capability / attribute caches.
#include <cmath>
#include <mutex>

#include "bsa.h"
#include "bsa_kernels.h"

namespace {

using bsa::Shape;

constexpr int kMaxN = 1 << 21;       // nb <= 16384 (bitmap / score tile sizes)
constexpr int kMaxBH = 65535;        // grid.y limit of the per-block kernels

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int shape_of(const bsa_params* p, Shape* s) {
  if (!p) return BSA_ERR_INVALID;
  if (p->D != 128 || p->B < 1 || p->H < 1 || p->N < 1 || p->N > kMaxN) return BSA_ERR_INVALID;
  if (static_cast<int64_t>(p->B) * p->H > kMaxBH) return BSA_ERR_INVALID;
  if (p->top_k < 1) return BSA_ERR_INVALID;
  if (p->prefix < 0 || p->prefix % 128 != 0 || p->prefix >= p->N) return BSA_ERR_INVALID;
  if (p->variant != BSA_SUMMARY_ANCHOR && p->variant != BSA_SUMMARY_MEAN) return BSA_ERR_INVALID;
  s->B = p->B;
  s->H = p->H;
  s->N = p->N;
  s->nb = (p->N + 127) / 128;
  s->pb = p->prefix / 128;
  s->nbv = s->nb - s->pb;
  s->k_eff = p->top_k < s->nbv ? p->top_k : s->nbv;
  s->kcap = p->prefix > 0 ? s->nb : s->pb + s->k_eff;
  s->variant = p->variant;
  s->prefix = p->prefix;
  s->dev_status = p->dev_status;
  return BSA_OK;
}

// The kernels use tcgen05 / TMA: sm_100 only.  Cached per device.
int check_device() {
  static std::mutex mu;
  static signed char ok[64];
  static bool init = false;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
  std::lock_guard<std::mutex> g(mu);
  if (!init) {
    for (auto& v : ok) v = -1;
    init = true;
  }
  if (dev >= 64) return BSA_ERR_UNSUPPORTED;
  if (ok[dev] < 0) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return BSA_ERR_CUDA;
    ok[dev] = (major == 10) ? 1 : 0;
  }
  return ok[dev] ? BSA_OK : BSA_ERR_UNSUPPORTED;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// bf16 [BH, rows, 128] viewed as a 3-D tensor; box = 64 columns (128 bytes,
// one swizzle atom) x 128 rows x 1 head.  Rows past `rows` read as zero.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t BH) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {128, rows, BH};
  const cuuint64_t strides[2] = {128 * 2, rows * 128 * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// bf16 [total_rows, 128] viewed as a 2-D tensor with a one-row box of 64
// columns (128 bytes, one swizzle atom): the map of row gathers
// (tile::gather4 brings four rows per instruction).
bool make_map_rows(CUtensorMap* m, const void* base, uint64_t total_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {128, total_rows};
  const cuuint64_t strides[1] = {128 * 2};
  const cuuint32_t box[2] = {64, 1};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// uint8 (e4m3 codes) [BH, rows, 128] viewed as a 3-D tensor; box = 128
// columns (128 bytes, one swizzle atom) x 128 rows x 1 head.
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t BH) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {128, rows, BH};
  const cuuint64_t strides[2] = {128, rows * 128};
  const cuuint32_t box[3] = {128, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// fp32 [BH, rows, 128] viewed as a 3-D tensor; box = 32 columns (128 bytes,
// one swizzle atom) x box_rows rows x 1 head.  Rows past `rows` read as zero.
bool make_map_f32(CUtensorMap* m, const void* base, uint64_t rows, uint64_t BH,
                  uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {128, rows, BH};
  const cuuint64_t strides[2] = {128 * 4, rows * 128 * 4};
  const cuuint32_t box[3] = {32, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// The pooled-score maps of the tensor-core selection, or NULL when the rows
// are too long for it (the SIMT kernel then runs) or a map cannot be made.
const bsa::SelectMaps* select_maps(const Shape& s, const float* qpool, const float* kpool,
                                   bsa::SelectMaps* m) {
  const int R = bsa::select_tc_rows(s);
  if (R <= 0) return nullptr;
  const uint64_t bh = static_cast<uint64_t>(s.B) * s.H;
  if (!make_map_f32(&m->q, qpool, s.nb, bh, static_cast<uint32_t>(R)) ||
      !make_map_f32(&m->k, kpool, s.nb, bh, 128))
    return nullptr;
  return m;
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// The FP8 operand set carved from one buffer in the order of
// bsa_fp8_operands (each piece 256-byte aligned); returns the bytes used.
size_t fp8_carve(const Shape& s, uint8_t* base, bsa::Fp8Operands* f) {
  const size_t bh = static_cast<size_t>(s.B) * s.H;
  const size_t ntile = (s.nb + 127) / 128;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* p = base ? base + off : nullptr;
    off += round256(bytes);
    return p;
  };
  uint8_t* q8 = take(bh * s.N * 128);
  uint8_t* qs = take(bh * s.nb * 4);
  uint8_t* k8 = take(bh * s.N * 128);
  uint8_t* ks = take(bh * s.nb * 4);
  uint8_t* vt8 = take(bh * s.nb * 128 * 128);
  uint8_t* vs = take(bh * s.nb * 4);
  uint8_t* ks8 = take(bh * s.nb * 128);
  uint8_t* kss = take(bh * ntile * 4);
  uint8_t* vst8 = take(bh * ntile * 128 * 128);
  uint8_t* vss = take(bh * ntile * 4);
  uint8_t* vref = take(bh * 4);
  if (f) {
    f->q8 = q8;
    f->q_scale = reinterpret_cast<float*>(qs);
    f->k8 = k8;
    f->k_scale = reinterpret_cast<float*>(ks);
    f->vt8 = vt8;
    f->v_scale = reinterpret_cast<float*>(vs);
    f->ks8 = ks8;
    f->ks_scale = reinterpret_cast<float*>(kss);
    f->vst8 = vst8;
    f->vs_scale = reinterpret_cast<float*>(vss);
    f->v_ref = reinterpret_cast<float*>(vref);
  }
  return off;
}

bsa::Fp8Operands from_abi(const bsa_fp8_operands& o) {
  return bsa::Fp8Operands{o.q8, o.q_scale, o.k8, o.k_scale, o.vt8, o.v_scale,
                          o.ks8, o.ks_scale, o.vst8, o.vs_scale, o.v_ref};
}

bool fp8_valid(const bsa_fp8_operands* o) {
  if (!o || !o->q8 || !o->q_scale || !o->k8 || !o->k_scale || !o->vt8 || !o->v_scale ||
      !o->ks8 || !o->ks_scale || !o->vst8 || !o->vs_scale || !o->v_ref)
    return false;
  return true;
}

bool fp8_aligned(const bsa_fp8_operands* o) {
  return aligned(o->q8, 16) && aligned(o->k8, 16) && aligned(o->vt8, 16) && aligned(o->ks8, 16) &&
         aligned(o->vst8, 16) && aligned(o->q_scale, 4) && aligned(o->k_scale, 4) &&
         aligned(o->v_scale, 4) && aligned(o->ks_scale, 4) && aligned(o->vs_scale, 4) &&
         aligned(o->v_ref, 4);
}

struct Workspace {
  float *qpool, *anchor, *kpool, *bias;
  void *ksum, *vsum;
  int32_t *idx, *cnt;
};

size_t carve(const Shape& s, uint8_t* base, Workspace* w) {
  const size_t bh = static_cast<size_t>(s.B) * s.H;
  const size_t blocks = bh * s.nb;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* p = base ? base + off : nullptr;
    off += round256(bytes);
    return p;
  };
  uint8_t* qpool = take(blocks * 128 * 4);
  uint8_t* anchor = take(bh * 128 * 4);
  uint8_t* kpool = take(blocks * 128 * 4);
  uint8_t* ksum = take(blocks * 128 * 2);
  uint8_t* vsum = take(blocks * 128 * 2);
  uint8_t* bias = take(blocks * 4);
  uint8_t* idx = take(blocks * static_cast<size_t>(s.kcap) * 4);
  uint8_t* cnt = take(blocks * 4);
  if (w) {
    w->qpool = reinterpret_cast<float*>(qpool);
    w->anchor = reinterpret_cast<float*>(anchor);
    w->kpool = reinterpret_cast<float*>(kpool);
    w->ksum = ksum;
    w->vsum = vsum;
    w->bias = reinterpret_cast<float*>(bias);
    w->idx = reinterpret_cast<int32_t*>(idx);
    w->cnt = reinterpret_cast<int32_t*>(cnt);
  }
  return off;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? BSA_OK : BSA_ERR_CUDA; }

int pool_impl(const Shape& s, const void* Q, float* qpool, float* anchor, cudaStream_t st) {
  return cuda_status(bsa::launch_pool(s, Q, qpool, anchor, st));
}
int summarize_impl(const Shape& s, const void* K, const void* V, const float* anchor, float* kpool,
                   void* ksum, void* vsum, float* bias, cudaStream_t st) {
  return cuda_status(bsa::launch_summarize(s, K, V, anchor, kpool, ksum, vsum, bias, st));
}
int select_impl(const Shape& s, const float* qpool, const float* kpool, int32_t* idx, int32_t* cnt,
                cudaStream_t st) {
  bsa::SelectMaps m;
  return cuda_status(bsa::launch_select(s, select_maps(s, qpool, kpool, &m), qpool, kpool, idx,
                                        cnt, st));
}
int attend_impl(const Shape& s, const void* Q, const void* K, const void* V, const int32_t* idx,
                const int32_t* cnt, const void* ksum, const void* vsum, const float* bias, void* O,
                float* lse, cudaStream_t st) {
  bsa::AttendMaps maps;
  const uint64_t bh = static_cast<uint64_t>(s.B) * s.H;
  if (!make_map(&maps.q, Q, s.N, bh) || !make_map(&maps.k, K, s.N, bh) ||
      !make_map(&maps.v, V, s.N, bh) || !make_map(&maps.ks, ksum, s.nb, bh) ||
      !make_map(&maps.vs, vsum, s.nb, bh))
    return BSA_ERR_UNSUPPORTED;
  return cuda_status(bsa::launch_attend(s, maps, idx, cnt, bias, O, lse, st));
}

int attend_lists_impl(const Shape& s, const void* Q, const void* K, const void* V,
                      const int32_t* idx, int kcap, const int32_t* cnt, const void* ksum,
                      const void* vsum, const float* bias, void* O, float* lse, void* scratch,
                      cudaStream_t st) {
  bsa::AttendMaps maps;
  const uint64_t bh = static_cast<uint64_t>(s.B) * s.H;
  if (!make_map(&maps.q, Q, s.N, bh) || !make_map(&maps.k, K, s.N, bh) ||
      !make_map(&maps.v, V, s.N, bh) || !make_map(&maps.ks, ksum, s.nb, bh) ||
      !make_map(&maps.vs, vsum, s.nb, bh))
    return BSA_ERR_UNSUPPORTED;
  return cuda_status(
      bsa::launch_attend_lists(s, maps, idx, kcap, cnt, bias, O, lse, scratch, st));
}

// The shape of a threshold call: list rows hold up to nb blocks.
Shape threshold_shape(const Shape& s) {
  Shape t = s;
  t.kcap = s.nb;
  return t;
}

// Reblocking scratch carved from one buffer (each piece 256-byte aligned).
size_t reblock_carve(const Shape& s, const bsa::ReblockPlan& plan, uint8_t* base,
                     bsa::ReblockBuffers* w) {
  const size_t bh = static_cast<size_t>(s.B) * s.H;
  const size_t nv = plan.nv;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* p = base ? base + off : nullptr;
    off += round256(bytes);
    return p;
  };
  uint8_t* perm_tmp = take(bh * s.N * 4);
  uint8_t* part = take(bh * plan.max_partials * 128 * 128 * 4);
  uint8_t* psum = take(bh * plan.max_partials * 128 * 4);
  uint8_t* vdir = take(bh * (static_cast<size_t>(1) << plan.levels) * 128 * 4);
  uint8_t* moment = take(bh * 128 * 128 * 4);
  uint8_t* r_hi = take(bh * 128 * 128 * 2);
  uint8_t* r_lo = take(bh * 128 * 128 * 2);
  uint8_t* u = take(bh * nv * 128 * 2);
  uint8_t* keys = take(bh * nv * 4);
  if (w) {
    w->perm_tmp = reinterpret_cast<int32_t*>(perm_tmp);
    w->part = reinterpret_cast<float*>(part);
    w->psum = reinterpret_cast<float*>(psum);
    w->vdir = reinterpret_cast<float*>(vdir);
    w->moment = reinterpret_cast<float*>(moment);
    w->r_hi = reinterpret_cast<__nv_bfloat16*>(r_hi);
    w->r_lo = reinterpret_cast<__nv_bfloat16*>(r_lo);
    w->u = reinterpret_cast<__nv_bfloat16*>(u);
    w->keys = reinterpret_cast<uint32_t*>(keys);
  }
  return off;
}

int reblock_impl(const Shape& s, const void* Q, const void* K, int32_t* perm, uint8_t* ws,
                 cudaStream_t st) {
  const bsa::ReblockPlan plan = bsa::reblock_plan(s);
  bsa::ReblockBuffers w;
  reblock_carve(s, plan, ws, &w);
  bsa::ReblockMaps maps;
  const uint64_t bh = static_cast<uint64_t>(s.B) * s.H;
  if (!make_map(&maps.q, Q, s.N, bh) || !make_map(&maps.r_hi, w.r_hi, 128, bh) ||
      !make_map(&maps.r_lo, w.r_lo, 128, bh))
    return BSA_ERR_UNSUPPORTED;
  // the whitened rows (only when there are video tokens to whiten)
  if (plan.nv > 0 && !make_map(&maps.u, w.u, static_cast<uint64_t>(plan.nv), bh))
    return BSA_ERR_UNSUPPORTED;
  return cuda_status(bsa::launch_reblock(s, plan, Q, K, maps, w, perm, st));
}

// Workspace of bsa_forward_reblock: perm, the permuted Q/K/V/O and lse, the
// reblocking scratch and the forward's own workspace.
struct ReblockForwardWs {
  int32_t* perm;
  void *Qp, *Kp, *Vp, *Op;
  float* lsep;
  uint8_t* rb;
  uint8_t* fw;
};

size_t reblock_forward_carve(const Shape& s, uint8_t* base, ReblockForwardWs* w) {
  const size_t bh = static_cast<size_t>(s.B) * s.H;
  const size_t rows = bh * s.N;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* p = base ? base + off : nullptr;
    off += round256(bytes);
    return p;
  };
  uint8_t* perm = take(rows * 4);
  uint8_t* qp = take(rows * 256);
  uint8_t* kp = take(rows * 256);
  uint8_t* vp = take(rows * 256);
  uint8_t* op = take(rows * 256);
  uint8_t* lsep = take(rows * 4);
  uint8_t* rb = take(reblock_carve(s, bsa::reblock_plan(s), nullptr, nullptr));
  uint8_t* fw = take(carve(s, nullptr, nullptr));
  if (w) *w = ReblockForwardWs{reinterpret_cast<int32_t*>(perm), qp, kp, vp, op,
                               reinterpret_cast<float*>(lsep), rb, fw};
  return off;
}

int quantize_fp8_impl(const Shape& s, const void* Q, const void* K, const void* V,
                      const void* ksum, const void* vsum, const bsa::Fp8Operands& f,
                      cudaStream_t st) {
  return cuda_status(bsa::launch_quantize_fp8(s, Q, K, V, ksum, vsum, f, st));
}

int attend_fp8_impl(const Shape& s, const bsa::Fp8Operands& f, const int32_t* idx,
                    const float* bias, void* O, float* lse, cudaStream_t st) {
  bsa::AttendMapsFp8 maps;
  const uint64_t bh = static_cast<uint64_t>(s.B) * s.H;
  const uint64_t ntile = (s.nb + 127) / 128;
  if (!make_map_u8(&maps.q, f.q8, s.N, bh) || !make_map_u8(&maps.k, f.k8, s.N, bh) ||
      !make_map_u8(&maps.vt, f.vt8, static_cast<uint64_t>(s.nb) * 128, bh) ||
      !make_map_u8(&maps.ks, f.ks8, s.nb, bh) ||
      !make_map_u8(&maps.vst, f.vst8, ntile * 128, bh))
    return BSA_ERR_UNSUPPORTED;
  return cuda_status(bsa::launch_attend_fp8(s, maps, f, idx, bias, O, lse, st));
}

// ------------------------------------------------------------ extra tokens

constexpr int kMaxExtra = BSA_MAX_EXTRA_TOKENS;

bool extra_valid(const Shape& s, int n_extra) {
  if (n_extra < 0 || n_extra > kMaxExtra) return false;
  // row coordinates of the gathers are 32-bit
  return static_cast<int64_t>(s.B) * s.H * s.N < (static_cast<int64_t>(1) << 31);
}

// Extra-token intermediates carved from one buffer (each piece 256-byte
// aligned): fp32 block statistics, the token lists, the side summary table
// and the candidate buffers of the selection.
struct ExtraWs {
  float *kstat, *vstat, *lse_blk;
  int32_t *extra, *ecnt;
  void *side_k, *side_v;
  float* side_bias;
  int32_t *side_blk, *side_cnt;
  void* cand;
};

size_t extra_carve(const Shape& s, int n_extra, uint8_t* base, ExtraWs* w) {
  const size_t bh = static_cast<size_t>(s.B) * s.H;
  const size_t blocks = bh * s.nb;
  const size_t scap = static_cast<size_t>(bsa::extra_side_cap(s, n_extra));
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* p = base ? base + off : nullptr;
    off += round256(bytes);
    return p;
  };
  uint8_t* kstat = take(blocks * 128 * 4);
  uint8_t* vstat = take(blocks * 128 * 4);
  uint8_t* lse_blk = take(blocks * 4);
  uint8_t* extra = take(blocks * static_cast<size_t>(n_extra) * 4);
  uint8_t* ecnt = take(blocks * 4);
  uint8_t* side_k = take(blocks * scap * 128 * 2);
  uint8_t* side_v = take(blocks * scap * 128 * 2);
  uint8_t* side_bias = take(blocks * scap * 4);
  uint8_t* side_blk = take(blocks * scap * 4);
  uint8_t* side_cnt = take(blocks * 4);
  uint8_t* cand = take(bsa::select_extra_scratch_bytes(s, n_extra));
  if (w) {
    w->kstat = reinterpret_cast<float*>(kstat);
    w->vstat = reinterpret_cast<float*>(vstat);
    w->lse_blk = reinterpret_cast<float*>(lse_blk);
    w->extra = reinterpret_cast<int32_t*>(extra);
    w->ecnt = reinterpret_cast<int32_t*>(ecnt);
    w->side_k = side_k;
    w->side_v = side_v;
    w->side_bias = reinterpret_cast<float*>(side_bias);
    w->side_blk = reinterpret_cast<int32_t*>(side_blk);
    w->side_cnt = reinterpret_cast<int32_t*>(side_cnt);
    w->cand = cand;
  }
  return off;
}

int select_extra_impl(const Shape& s, int n_extra, const float* qpool, const void* K,
                      const int32_t* idx, const int32_t* cnt, int32_t* extra, int32_t* ecnt,
                      void* scratch, cudaStream_t st) {
  const size_t blocks = static_cast<size_t>(s.B) * s.H * s.nb;
  if (n_extra == 0) return cuda_status(cudaMemsetAsync(ecnt, 0, blocks * 4, st));
  CUtensorMap tm_k;
  if (!make_map(&tm_k, K, s.N, static_cast<uint64_t>(s.B) * s.H)) return BSA_ERR_UNSUPPORTED;
  return cuda_status(bsa::launch_select_extra(s, n_extra, tm_k, qpool, idx, s.kcap, cnt, extra,
                                              ecnt, scratch, st));
}

int extra_summaries_impl(const Shape& s, int n_extra, const void* K, const void* V,
                         const float* anchor, const float* kpool, const float* kstat,
                         const float* vstat, const float* lse_blk, const int32_t* extra,
                         const int32_t* ecnt, void* side_k, void* side_v, float* side_bias,
                         int32_t* side_blk, int32_t* side_cnt, cudaStream_t st) {
  const size_t blocks = static_cast<size_t>(s.B) * s.H * s.nb;
  // prefix query blocks have no side rows
  cudaError_t e = cudaMemsetAsync(side_cnt, 0, blocks * 4, st);
  if (e != cudaSuccess || n_extra == 0) return cuda_status(e);
  return cuda_status(bsa::launch_extra_summaries(s, n_extra, K, V, anchor, kpool, kstat, vstat,
                                                 lse_blk, extra, ecnt, side_k, side_v, side_bias,
                                                 side_blk, side_cnt, st));
}

int attend_extra_impl(const Shape& s, int n_extra, const void* Q, const void* K, const void* V,
                      const int32_t* idx, const int32_t* extra, const int32_t* ecnt,
                      const void* ksum, const void* vsum, const float* bias, const void* side_k,
                      const void* side_v, const float* side_bias, const int32_t* side_cnt,
                      void* O, float* lse, cudaStream_t st) {
  bsa::AttendMaps maps;
  bsa::AttendExtraMaps xm;
  const uint64_t bh = static_cast<uint64_t>(s.B) * s.H;
  const int scap = bsa::extra_side_cap(s, n_extra);
  if (!make_map(&maps.q, Q, s.N, bh) || !make_map(&maps.k, K, s.N, bh) ||
      !make_map(&maps.v, V, s.N, bh) || !make_map(&maps.ks, ksum, s.nb, bh) ||
      !make_map(&maps.vs, vsum, s.nb, bh) || !make_map_rows(&xm.k2, K, bh * s.N) ||
      !make_map_rows(&xm.v2, V, bh * s.N))
    return BSA_ERR_UNSUPPORTED;
  if (scap > 0) {
    const uint64_t rows = static_cast<uint64_t>(s.nb) * scap;
    if (!make_map(&xm.sk, side_k, rows, bh) || !make_map(&xm.sv, side_v, rows, bh))
      return BSA_ERR_UNSUPPORTED;
  } else {   // never read: no row has side summaries
    xm.sk = maps.ks;
    xm.sv = maps.vs;
  }
  return cuda_status(bsa::launch_attend_extra(s, maps, xm, idx, extra, ecnt, n_extra, bias,
                                              side_bias, side_cnt, scap, O, lse, st));
}

// A forward from HOST buffers, pipelined over up to `max_chunks` chunks of
// (b, h) slices; `fwd` runs the forward of one chunk (a sub-call with B = 1)
// on the caller's stream with the caller's workspace, which a sub-call needs
// no more of than the whole call.  Validates the pointers of the device side
// before the first copy, so an argument error enqueues nothing.
constexpr int kMaxChunks = 16;
template <class Fwd>
int forward_host_pipelined(const bsa_params* p, const void* hQ, const void* hK, const void* hV,
                           void* hO, float* hlse, void* dQ, void* dK, void* dV, void* dO,
                           float* dlse, void* workspace, size_t workspace_bytes, void* stream,
                           Fwd fwd, int max_chunks = kMaxChunks) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!hQ || !hK || !hV || !hO) return BSA_ERR_INVALID;
  if (!dQ || !dK || !dV || !dO || !workspace) return BSA_ERR_INVALID;
  if (!aligned(dQ, 16) || !aligned(dK, 16) || !aligned(dV, 16) || !aligned(dO, 16) ||
      !aligned(workspace, 256) || (dlse && !aligned(dlse, 4)))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;

  // Pipeline over chunks of (b, h) slices (every slice is independent):
  // host->device copies on one helper stream, the forward on the caller's
  // stream, device->host copies on another helper stream, ordered by events.
  // Copies of chunk c+1 overlap the forward of chunk c, and the two copy
  // directions overlap each other.  The helper streams and events are made
  // per call and released when their work is done; the caller's stream
  // waits for the last copy, so synchronising it covers everything.
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = s.B * s.H;
  // up to 16 chunks by default: the last chunk's forward and copy back are
  // what the pipeline cannot hide (measured at 56 heads: 33.5 / 119.6 ms with
  // 8 chunks, 32.9 / 115.8 with 14 of 4 heads, 33.2 / 114.3 with 28 of 2, for
  // 768p-5s / 2K-5s)
  const int cap = max_chunks < 1 ? 1 : (max_chunks > kMaxChunks ? kMaxChunks : max_chunks);
  const int nchunk = BH < cap ? BH : cap;
  const int per = (BH + nchunk - 1) / nchunk;
  const size_t slice = static_cast<size_t>(s.N) * 128 * 2;     // bytes of one (b, h) slice
  const size_t lslice = static_cast<size_t>(s.N) * 4;
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t ev_start = nullptr, ev_done = nullptr, ev_in[kMaxChunks] = {},
              ev_comp[kMaxChunks] = {};
  auto cleanup = [&]() {
    for (int c = 0; c < kMaxChunks; ++c) {
      if (ev_in[c]) cudaEventDestroy(ev_in[c]);
      if (ev_comp[c]) cudaEventDestroy(ev_comp[c]);
    }
    if (ev_start) cudaEventDestroy(ev_start);
    if (ev_done) cudaEventDestroy(ev_done);
    if (s_in) cudaStreamDestroy(s_in);
    if (s_out) cudaStreamDestroy(s_out);
  };
  bool ok = cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&ev_start, cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&ev_done, cudaEventDisableTiming) == cudaSuccess;
  for (int c = 0; ok && c < nchunk; ++c)
    ok = cudaEventCreateWithFlags(&ev_in[c], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&ev_comp[c], cudaEventDisableTiming) == cudaSuccess;
  // helper streams start after earlier work on the caller's stream
  ok = ok && cudaEventRecord(ev_start, st) == cudaSuccess &&
       cudaStreamWaitEvent(s_in, ev_start, 0) == cudaSuccess &&
       cudaStreamWaitEvent(s_out, ev_start, 0) == cudaSuccess;
  if (!ok) {
    cleanup();
    return BSA_ERR_CUDA;
  }
  auto off = [](const void* base, size_t bytes) {
    return static_cast<const char*>(base) + bytes;
  };
  for (int c = 0; c < nchunk && rc == BSA_OK; ++c) {
    const int bh0 = c * per;
    const int nbh = (BH - bh0) < per ? (BH - bh0) : per;
    if (nbh <= 0) break;
    const size_t o = static_cast<size_t>(bh0) * slice, bytes = static_cast<size_t>(nbh) * slice;
    char* q = static_cast<char*>(dQ) + o;
    char* k = static_cast<char*>(dK) + o;
    char* v = static_cast<char*>(dV) + o;
    char* out = static_cast<char*>(dO) + o;
    float* l = dlse ? dlse + static_cast<size_t>(bh0) * s.N : nullptr;
    if (cudaMemcpyAsync(q, off(hQ, o), bytes, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaMemcpyAsync(k, off(hK, o), bytes, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaMemcpyAsync(v, off(hV, o), bytes, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaEventRecord(ev_in[c], s_in) != cudaSuccess ||
        cudaStreamWaitEvent(st, ev_in[c], 0) != cudaSuccess) {
      rc = BSA_ERR_CUDA;
      break;
    }
    bsa_params sub = *p;
    sub.B = 1;
    sub.H = nbh;
    if ((rc = fwd(&sub, q, k, v, out, l, workspace, workspace_bytes, stream))) break;
    if (cudaEventRecord(ev_comp[c], st) != cudaSuccess ||
        cudaStreamWaitEvent(s_out, ev_comp[c], 0) != cudaSuccess ||
        cudaMemcpyAsync(static_cast<char*>(hO) + o, out, bytes, cudaMemcpyDeviceToHost, s_out) !=
            cudaSuccess ||
        (hlse && l &&
         cudaMemcpyAsync(hlse + static_cast<size_t>(bh0) * s.N, l, nbh * lslice,
                         cudaMemcpyDeviceToHost, s_out) != cudaSuccess)) {
      rc = BSA_ERR_CUDA;
      break;
    }
  }
  // the caller's stream waits for the last copy back
  if (cudaEventRecord(ev_done, s_out) != cudaSuccess || cudaStreamWaitEvent(st, ev_done, 0) != cudaSuccess)
    rc = rc ? rc : BSA_ERR_CUDA;
  cleanup();
  return rc;
}

}  // namespace

extern "C" {

int32_t bsa_extra_side_capacity(const bsa_params* p, int32_t n_extra) {
  Shape s;
  if (shape_of(p, &s) != BSA_OK || !extra_valid(s, n_extra)) return -1;
  return bsa::extra_side_cap(s, n_extra);
}

int bsa_summarize_stats(const bsa_params* p, const void* K, const void* V, const float* anchor,
                        float* kpool, void* ksum, void* vsum, float* bias, float* kstat,
                        float* vstat, float* lse_blk, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!K || !V || !kpool || !ksum || !vsum || !bias || !kstat || !vstat || !lse_blk)
    return BSA_ERR_INVALID;
  if (s.variant == BSA_SUMMARY_ANCHOR && !anchor) return BSA_ERR_INVALID;
  if (!aligned(K, 16) || !aligned(V, 16) || !aligned(kpool, 16) || !aligned(ksum, 16) ||
      !aligned(vsum, 16) || !aligned(bias, 4) || (anchor && !aligned(anchor, 16)) ||
      !aligned(kstat, 16) || !aligned(vstat, 16) || !aligned(lse_blk, 4))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return cuda_status(bsa::launch_summarize(s, K, V, anchor, kpool, ksum, vsum, bias,
                                           static_cast<cudaStream_t>(stream), kstat, vstat,
                                           lse_blk));
}

size_t bsa_select_extra_workspace_bytes(const bsa_params* p, int32_t n_extra) {
  Shape s;
  if (shape_of(p, &s) != BSA_OK || !extra_valid(s, n_extra)) return 0;
  return bsa::select_extra_scratch_bytes(s, n_extra);
}

int bsa_select_extra(const bsa_params* p, int32_t n_extra, const float* qpool, const void* K,
                     const int32_t* idx, const int32_t* cnt, int32_t* extra, int32_t* ecnt,
                     void* workspace, size_t workspace_bytes, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!extra_valid(s, n_extra)) return BSA_ERR_INVALID;
  if (!qpool || !K || !idx || !cnt || !ecnt || (n_extra > 0 && (!extra || !workspace)))
    return BSA_ERR_INVALID;
  if (workspace_bytes < bsa::select_extra_scratch_bytes(s, n_extra)) return BSA_ERR_INVALID;
  if (!aligned(qpool, 16) || !aligned(K, 16) || !aligned(idx, 4) || !aligned(cnt, 4) ||
      !aligned(extra, 4) || !aligned(ecnt, 4) || !aligned(workspace, 256))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return select_extra_impl(s, n_extra, qpool, K, idx, cnt, extra, ecnt, workspace,
                           static_cast<cudaStream_t>(stream));
}

int bsa_extra_summaries(const bsa_params* p, int32_t n_extra, const void* K, const void* V,
                        const float* anchor, const float* kpool, const float* kstat,
                        const float* vstat, const float* lse_blk, const int32_t* extra,
                        const int32_t* ecnt, void* side_k, void* side_v, float* side_bias,
                        int32_t* side_blk, int32_t* side_cnt, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!extra_valid(s, n_extra)) return BSA_ERR_INVALID;
  if (!K || !V || !kpool || !kstat || !vstat || !lse_blk || !ecnt || !side_cnt)
    return BSA_ERR_INVALID;
  if (s.variant == BSA_SUMMARY_ANCHOR && !anchor) return BSA_ERR_INVALID;
  if (n_extra > 0 && (!extra || !side_k || !side_v || !side_bias || !side_blk))
    return BSA_ERR_INVALID;
  if (!aligned(K, 16) || !aligned(V, 16) || (anchor && !aligned(anchor, 16)) ||
      !aligned(kpool, 16) || !aligned(kstat, 16) || !aligned(vstat, 16) || !aligned(lse_blk, 4) ||
      !aligned(extra, 4) || !aligned(ecnt, 4) || !aligned(side_k, 16) || !aligned(side_v, 16) ||
      !aligned(side_bias, 4) || !aligned(side_blk, 4) || !aligned(side_cnt, 4))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return extra_summaries_impl(s, n_extra, K, V, anchor, kpool, kstat, vstat, lse_blk, extra, ecnt,
                              side_k, side_v, side_bias, side_blk, side_cnt,
                              static_cast<cudaStream_t>(stream));
}

int bsa_attend_extra(const bsa_params* p, int32_t n_extra, const void* Q, const void* K,
                     const void* V, const int32_t* idx, const int32_t* cnt, const int32_t* extra,
                     const int32_t* ecnt, const void* ksum, const void* vsum, const float* bias,
                     const void* side_k, const void* side_v, const float* side_bias,
                     const int32_t* side_cnt, void* O, float* lse, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!extra_valid(s, n_extra)) return BSA_ERR_INVALID;
  if (!Q || !K || !V || !idx || !cnt || !ecnt || !ksum || !vsum || !bias || !side_cnt || !O)
    return BSA_ERR_INVALID;
  if (n_extra > 0 && (!extra || !side_k || !side_v || !side_bias)) return BSA_ERR_INVALID;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(ksum, 16) ||
      !aligned(vsum, 16) || !aligned(O, 16) || !aligned(idx, 4) || !aligned(cnt, 4) ||
      !aligned(extra, 4) || !aligned(ecnt, 4) || !aligned(bias, 4) || !aligned(side_k, 16) ||
      !aligned(side_v, 16) || !aligned(side_bias, 4) || !aligned(side_cnt, 4) ||
      (lse && !aligned(lse, 4)))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return attend_extra_impl(s, n_extra, Q, K, V, idx, extra, ecnt, ksum, vsum, bias, side_k, side_v,
                           side_bias, side_cnt, O, lse, static_cast<cudaStream_t>(stream));
}

size_t bsa_forward_extra_workspace_bytes(const bsa_params* p, int32_t n_extra) {
  Shape s;
  if (shape_of(p, &s) != BSA_OK || !extra_valid(s, n_extra)) return 0;
  return carve(s, nullptr, nullptr) + extra_carve(s, n_extra, nullptr, nullptr);
}

int bsa_forward_extra(const bsa_params* p, int32_t n_extra, const void* Q, const void* K,
                      const void* V, void* O, float* lse, void* workspace, size_t workspace_bytes,
                      void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!extra_valid(s, n_extra)) return BSA_ERR_INVALID;
  if (!Q || !K || !V || !O || !workspace) return BSA_ERR_INVALID;
  const size_t ws0 = carve(s, nullptr, nullptr);
  if (workspace_bytes < ws0 + extra_carve(s, n_extra, nullptr, nullptr)) return BSA_ERR_INVALID;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16) ||
      !aligned(workspace, 256) || (lse && !aligned(lse, 4)))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  Workspace w;
  carve(s, static_cast<uint8_t*>(workspace), &w);
  ExtraWs x;
  extra_carve(s, n_extra, static_cast<uint8_t*>(workspace) + ws0, &x);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = pool_impl(s, Q, w.qpool, w.anchor, st))) return rc;
  if ((rc = cuda_status(bsa::launch_summarize(s, K, V, w.anchor, w.kpool, w.ksum, w.vsum, w.bias,
                                              st, x.kstat, x.vstat, x.lse_blk))))
    return rc;
  if ((rc = select_impl(s, w.qpool, w.kpool, w.idx, w.cnt, st))) return rc;
  if ((rc = select_extra_impl(s, n_extra, w.qpool, K, w.idx, w.cnt, x.extra, x.ecnt, x.cand, st)))
    return rc;
  if ((rc = extra_summaries_impl(s, n_extra, K, V, w.anchor, w.kpool, x.kstat, x.vstat, x.lse_blk,
                                 x.extra, x.ecnt, x.side_k, x.side_v, x.side_bias, x.side_blk,
                                 x.side_cnt, st)))
    return rc;
  return attend_extra_impl(s, n_extra, Q, K, V, w.idx, x.extra, x.ecnt, w.ksum, w.vsum, w.bias,
                           x.side_k, x.side_v, x.side_bias, x.side_cnt, O, lse, st);
}

size_t bsa_reblock_workspace_bytes(const bsa_params* p) {
  Shape s;
  if (shape_of(p, &s) != BSA_OK) return 0;
  return reblock_carve(s, bsa::reblock_plan(s), nullptr, nullptr);
}

int bsa_reblock(const bsa_params* p, const void* Q, const void* K, int32_t* perm,
                void* workspace, size_t workspace_bytes, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!Q || !K || !perm || !workspace) return BSA_ERR_INVALID;
  if (workspace_bytes < reblock_carve(s, bsa::reblock_plan(s), nullptr, nullptr))
    return BSA_ERR_INVALID;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(perm, 4) || !aligned(workspace, 256))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return reblock_impl(s, Q, K, perm, static_cast<uint8_t*>(workspace),
                      static_cast<cudaStream_t>(stream));
}

int bsa_permute(const bsa_params* p, const void* Q, const void* K, const void* V,
                const int32_t* perm, void* Qp, void* Kp, void* Vp, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!Q || !K || !V || !perm || !Qp || !Kp || !Vp) return BSA_ERR_INVALID;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(Qp, 16) ||
      !aligned(Kp, 16) || !aligned(Vp, 16) || !aligned(perm, 4))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return cuda_status(bsa::launch_permute_rows(s, Q, K, V, perm, Qp, Kp, Vp,
                                              static_cast<cudaStream_t>(stream)));
}

int bsa_pool_permuted(const bsa_params* p, const void* Q, const int32_t* perm, void* Qp,
                      float* qpool, float* anchor, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!Q || !perm || !Qp || !qpool || !anchor) return BSA_ERR_INVALID;
  if (!aligned(Q, 16) || !aligned(Qp, 16) || !aligned(perm, 4) || !aligned(qpool, 16) ||
      !aligned(anchor, 16))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return cuda_status(
      bsa::launch_pool(s, Q, qpool, anchor, static_cast<cudaStream_t>(stream), perm, Qp));
}

int bsa_summarize_permuted(const bsa_params* p, const void* K, const void* V,
                           const int32_t* perm, void* Kp, void* Vp, const float* anchor,
                           float* kpool, void* ksum, void* vsum, float* bias, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!K || !V || !perm || !Kp || !Vp || !kpool || !ksum || !vsum || !bias) return BSA_ERR_INVALID;
  if (s.variant == BSA_SUMMARY_ANCHOR && !anchor) return BSA_ERR_INVALID;
  if (!aligned(K, 16) || !aligned(V, 16) || !aligned(Kp, 16) || !aligned(Vp, 16) ||
      !aligned(perm, 4) || !aligned(kpool, 16) || !aligned(ksum, 16) || !aligned(vsum, 16) ||
      !aligned(bias, 4) || (anchor && !aligned(anchor, 16)))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return cuda_status(bsa::launch_summarize(s, K, V, anchor, kpool, ksum, vsum, bias,
                                           static_cast<cudaStream_t>(stream), nullptr, nullptr,
                                           nullptr, perm, Kp, Vp));
}

int bsa_unpermute(const bsa_params* p, const void* Op, const float* lsep, const int32_t* perm,
                  void* O, float* lse, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!Op || !perm || !O || (lse && !lsep)) return BSA_ERR_INVALID;
  if (!aligned(Op, 16) || !aligned(O, 16) || !aligned(perm, 4) || (lse && !aligned(lse, 4)) ||
      (lsep && !aligned(lsep, 4)))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return cuda_status(bsa::launch_unpermute_rows(s, Op, lse ? lsep : nullptr, perm, O, lse,
                                                static_cast<cudaStream_t>(stream)));
}

size_t bsa_forward_reblock_workspace_bytes(const bsa_params* p) {
  Shape s;
  if (shape_of(p, &s) != BSA_OK) return 0;
  return reblock_forward_carve(s, nullptr, nullptr);
}

int bsa_forward_reblock(const bsa_params* p, const void* Q, const void* K, const void* V,
                        void* O, float* lse, void* workspace, size_t workspace_bytes,
                        void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!Q || !K || !V || !O || !workspace) return BSA_ERR_INVALID;
  if (workspace_bytes < reblock_forward_carve(s, nullptr, nullptr)) return BSA_ERR_INVALID;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16) ||
      !aligned(workspace, 256) || (lse && !aligned(lse, 4)))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  ReblockForwardWs w;
  reblock_forward_carve(s, static_cast<uint8_t*>(workspace), &w);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = reblock_impl(s, Q, K, w.perm, w.rb, st))) return rc;
  Workspace fw;
  carve(s, w.fw, &fw);
  // pool and summarize read Q, K, V through the permutation and write the
  // permuted rows the attention reads (no separate gather pass)
  if ((rc = cuda_status(bsa::launch_pool(s, Q, fw.qpool, fw.anchor, st, w.perm, w.Qp))))
    return rc;
  if ((rc = cuda_status(bsa::launch_summarize(s, K, V, fw.anchor, fw.kpool, fw.ksum, fw.vsum,
                                              fw.bias, st, nullptr, nullptr, nullptr, w.perm,
                                              w.Kp, w.Vp))))
    return rc;
  if ((rc = select_impl(s, fw.qpool, fw.kpool, fw.idx, fw.cnt, st))) return rc;
  if ((rc = attend_impl(s, w.Qp, w.Kp, w.Vp, fw.idx, fw.cnt, fw.ksum, fw.vsum, fw.bias, w.Op,
                        lse ? w.lsep : nullptr, st)))
    return rc;
  return cuda_status(
      bsa::launch_unpermute_rows(s, w.Op, lse ? w.lsep : nullptr, w.perm, O, lse, st));
}

size_t bsa_fp8_operands_bytes(const bsa_params* p) {
  Shape s;
  if (shape_of(p, &s) != BSA_OK) return 0;
  return fp8_carve(s, nullptr, nullptr);
}

int bsa_fp8_operands_carve(const bsa_params* p, void* base, size_t bytes, bsa_fp8_operands* out) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!base || !out || bytes < fp8_carve(s, nullptr, nullptr)) return BSA_ERR_INVALID;
  if (!aligned(base, 256)) return BSA_ERR_ALIGN;
  bsa::Fp8Operands f;
  fp8_carve(s, static_cast<uint8_t*>(base), &f);
  *out = bsa_fp8_operands{f.q8, f.q_scale, f.k8, f.k_scale, f.vt8, f.v_scale,
                          f.ks8, f.ks_scale, f.vst8, f.vs_scale, f.v_ref};
  return BSA_OK;
}

int bsa_quantize_fp8(const bsa_params* p, const void* Q, const void* K, const void* V,
                     const void* ksum, const void* vsum, const bsa_fp8_operands* ops,
                     void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!Q || !K || !V || !ksum || !vsum || !fp8_valid(ops)) return BSA_ERR_INVALID;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(ksum, 16) ||
      !aligned(vsum, 16) || !fp8_aligned(ops))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return quantize_fp8_impl(s, Q, K, V, ksum, vsum, from_abi(*ops),
                           static_cast<cudaStream_t>(stream));
}

int bsa_attend_fp8(const bsa_params* p, const bsa_fp8_operands* ops, const int32_t* idx,
                   const int32_t* cnt, const float* bias, void* O, float* lse, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!fp8_valid(ops) || !idx || !cnt || !bias || !O) return BSA_ERR_INVALID;
  if (!fp8_aligned(ops) || !aligned(O, 16) || !aligned(idx, 4) || !aligned(cnt, 4) ||
      !aligned(bias, 4) || (lse && !aligned(lse, 4)))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return attend_fp8_impl(s, from_abi(*ops), idx, bias, O, lse, static_cast<cudaStream_t>(stream));
}

size_t bsa_forward_fp8_workspace_bytes(const bsa_params* p) {
  Shape s;
  if (shape_of(p, &s) != BSA_OK) return 0;
  return carve(s, nullptr, nullptr) + fp8_carve(s, nullptr, nullptr);
}

int bsa_forward_fp8(const bsa_params* p, const void* Q, const void* K, const void* V, void* O,
                    float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!Q || !K || !V || !O || !workspace) return BSA_ERR_INVALID;
  const size_t ws0 = carve(s, nullptr, nullptr);
  if (workspace_bytes < ws0 + fp8_carve(s, nullptr, nullptr)) return BSA_ERR_INVALID;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16) ||
      !aligned(workspace, 256) || (lse && !aligned(lse, 4)))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  Workspace w;
  carve(s, static_cast<uint8_t*>(workspace), &w);
  bsa::Fp8Operands f;
  fp8_carve(s, static_cast<uint8_t*>(workspace) + ws0, &f);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = pool_impl(s, Q, w.qpool, w.anchor, st))) return rc;
  if ((rc = summarize_impl(s, K, V, w.anchor, w.kpool, w.ksum, w.vsum, w.bias, st))) return rc;
  if ((rc = select_impl(s, w.qpool, w.kpool, w.idx, w.cnt, st))) return rc;
  if ((rc = quantize_fp8_impl(s, Q, K, V, w.ksum, w.vsum, f, st))) return rc;
  return attend_fp8_impl(s, f, w.idx, w.bias, O, lse, st);
}

int32_t bsa_threshold_capacity(const bsa_params* p) {
  Shape s;
  return shape_of(p, &s) == BSA_OK ? s.nb : -1;
}

int bsa_select_threshold(const bsa_params* p, float tau, const float* qpool, const float* kpool,
                         int32_t* idx, int32_t* cnt, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!std::isfinite(tau) || !qpool || !kpool || !idx || !cnt) return BSA_ERR_INVALID;
  if (!aligned(qpool, 16) || !aligned(kpool, 16) || !aligned(idx, 4) || !aligned(cnt, 4))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  bsa::SelectMaps m;
  return cuda_status(bsa::launch_select_threshold(s, tau, select_maps(s, qpool, kpool, &m), qpool,
                                                  kpool, idx, cnt,
                                                  static_cast<cudaStream_t>(stream)));
}

size_t bsa_attend_lists_workspace_bytes(const bsa_params* p) {
  Shape s;
  if (shape_of(p, &s) != BSA_OK) return 0;
  return bsa::attend_lists_scratch_bytes(s);
}

int bsa_attend_lists(const bsa_params* p, const void* Q, const void* K, const void* V,
                     const int32_t* idx, int32_t kcap, const int32_t* cnt, const void* ksum,
                     const void* vsum, const float* bias, void* O, float* lse, void* workspace,
                     size_t workspace_bytes, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!Q || !K || !V || !idx || !cnt || !ksum || !vsum || !bias || !O || !workspace)
    return BSA_ERR_INVALID;
  // prefix rows list all nb blocks, so a row must have room for them
  if (kcap < (s.pb > 0 ? s.nb : 1) || kcap > s.nb) return BSA_ERR_INVALID;
  if (workspace_bytes < bsa::attend_lists_scratch_bytes(s)) return BSA_ERR_INVALID;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(ksum, 16) ||
      !aligned(vsum, 16) || !aligned(O, 16) || !aligned(idx, 4) || !aligned(cnt, 4) ||
      !aligned(bias, 4) || !aligned(workspace, 256) || (lse && !aligned(lse, 4)))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return attend_lists_impl(s, Q, K, V, idx, kcap, cnt, ksum, vsum, bias, O, lse, workspace,
                           static_cast<cudaStream_t>(stream));
}

size_t bsa_forward_threshold_workspace_bytes(const bsa_params* p) {
  Shape s;
  if (shape_of(p, &s) != BSA_OK) return 0;
  return carve(threshold_shape(s), nullptr, nullptr) + bsa::attend_lists_scratch_bytes(s);
}

int bsa_forward_threshold(const bsa_params* p, float tau, const void* Q, const void* K,
                          const void* V, void* O, float* lse, void* workspace,
                          size_t workspace_bytes, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!std::isfinite(tau) || !Q || !K || !V || !O || !workspace) return BSA_ERR_INVALID;
  const Shape t = threshold_shape(s);
  const size_t ws0 = carve(t, nullptr, nullptr);
  if (workspace_bytes < ws0 + bsa::attend_lists_scratch_bytes(s)) return BSA_ERR_INVALID;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16) ||
      !aligned(workspace, 256) || (lse && !aligned(lse, 4)))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  Workspace w;
  carve(t, static_cast<uint8_t*>(workspace), &w);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = pool_impl(s, Q, w.qpool, w.anchor, st))) return rc;
  if ((rc = summarize_impl(s, K, V, w.anchor, w.kpool, w.ksum, w.vsum, w.bias, st))) return rc;
  bsa::SelectMaps m;
  if ((rc = cuda_status(bsa::launch_select_threshold(
           s, tau, select_maps(s, w.qpool, w.kpool, &m), w.qpool, w.kpool, w.idx, w.cnt, st))))
    return rc;
  return attend_lists_impl(s, Q, K, V, w.idx, s.nb, w.cnt, w.ksum, w.vsum, w.bias, O, lse,
                           static_cast<uint8_t*>(workspace) + ws0, st);
}

int32_t bsa_num_blocks(const bsa_params* p) {
  Shape s;
  return shape_of(p, &s) == BSA_OK ? s.nb : -1;
}

int32_t bsa_select_capacity(const bsa_params* p) {
  Shape s;
  return shape_of(p, &s) == BSA_OK ? s.kcap : -1;
}

size_t bsa_workspace_bytes(const bsa_params* p) {
  Shape s;
  if (shape_of(p, &s) != BSA_OK) return 0;
  return carve(s, nullptr, nullptr);
}

int bsa_pool(const bsa_params* p, const void* Q, float* qpool, float* anchor, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!Q || !qpool || !anchor) return BSA_ERR_INVALID;
  if (!aligned(Q, 16) || !aligned(qpool, 16) || !aligned(anchor, 16)) return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return pool_impl(s, Q, qpool, anchor, static_cast<cudaStream_t>(stream));
}

int bsa_summarize(const bsa_params* p, const void* K, const void* V, const float* anchor,
                  float* kpool, void* ksum, void* vsum, float* bias, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!K || !V || !kpool || !ksum || !vsum || !bias) return BSA_ERR_INVALID;
  if (s.variant == BSA_SUMMARY_ANCHOR && !anchor) return BSA_ERR_INVALID;
  if (!aligned(K, 16) || !aligned(V, 16) || !aligned(kpool, 16) || !aligned(ksum, 16) ||
      !aligned(vsum, 16) || !aligned(bias, 4) || (anchor && !aligned(anchor, 16)))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return summarize_impl(s, K, V, anchor, kpool, ksum, vsum, bias, static_cast<cudaStream_t>(stream));
}

int bsa_select(const bsa_params* p, const float* qpool, const float* kpool, int32_t* idx,
               int32_t* cnt, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!qpool || !kpool || !idx || !cnt) return BSA_ERR_INVALID;
  if (!aligned(qpool, 16) || !aligned(kpool, 16) || !aligned(idx, 4) || !aligned(cnt, 4))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return select_impl(s, qpool, kpool, idx, cnt, static_cast<cudaStream_t>(stream));
}

int bsa_attend(const bsa_params* p, const void* Q, const void* K, const void* V,
               const int32_t* idx, const int32_t* cnt, const void* ksum, const void* vsum,
               const float* bias, void* O, float* lse, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!Q || !K || !V || !idx || !cnt || !ksum || !vsum || !bias || !O) return BSA_ERR_INVALID;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(ksum, 16) ||
      !aligned(vsum, 16) || !aligned(O, 16) || !aligned(idx, 4) || !aligned(cnt, 4) ||
      !aligned(bias, 4) || (lse && !aligned(lse, 4)))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  return attend_impl(s, Q, K, V, idx, cnt, ksum, vsum, bias, O, lse,
                     static_cast<cudaStream_t>(stream));
}

int bsa_forward(const bsa_params* p, const void* Q, const void* K, const void* V, void* O,
                float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!Q || !K || !V || !O || !workspace) return BSA_ERR_INVALID;
  if (workspace_bytes < carve(s, nullptr, nullptr)) return BSA_ERR_INVALID;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16) ||
      !aligned(workspace, 256) || (lse && !aligned(lse, 4)))
    return BSA_ERR_ALIGN;
  if ((rc = check_device())) return rc;
  Workspace w;
  carve(s, static_cast<uint8_t*>(workspace), &w);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = pool_impl(s, Q, w.qpool, w.anchor, st))) return rc;
  if ((rc = summarize_impl(s, K, V, w.anchor, w.kpool, w.ksum, w.vsum, w.bias, st))) return rc;
  if ((rc = select_impl(s, w.qpool, w.kpool, w.idx, w.cnt, st))) return rc;
  return attend_impl(s, Q, K, V, w.idx, w.cnt, w.ksum, w.vsum, w.bias, O, lse, st);
}

int bsa_forward_host(const bsa_params* p, const void* hQ, const void* hK, const void* hV,
                     void* hO, float* hlse, void* dQ, void* dK, void* dV, void* dO, float* dlse,
                     void* workspace, size_t workspace_bytes, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (workspace_bytes < carve(s, nullptr, nullptr)) return BSA_ERR_INVALID;
  return forward_host_pipelined(
      p, hQ, hK, hV, hO, hlse, dQ, dK, dV, dO, dlse, workspace, workspace_bytes, stream,
      [](const bsa_params* sub, void* q, void* k, void* v, void* o, float* l, void* ws,
         size_t wsb, void* st) { return bsa_forward(sub, q, k, v, o, l, ws, wsb, st); });
}

int bsa_forward_fp8_host(const bsa_params* p, const void* hQ, const void* hK, const void* hV,
                         void* hO, float* hlse, void* dQ, void* dK, void* dV, void* dO,
                         float* dlse, void* workspace, size_t workspace_bytes, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (workspace_bytes < carve(s, nullptr, nullptr) + fp8_carve(s, nullptr, nullptr))
    return BSA_ERR_INVALID;
  return forward_host_pipelined(
      p, hQ, hK, hV, hO, hlse, dQ, dK, dV, dO, dlse, workspace, workspace_bytes, stream,
      [](const bsa_params* sub, void* q, void* k, void* v, void* o, float* l, void* ws,
         size_t wsb, void* st) { return bsa_forward_fp8(sub, q, k, v, o, l, ws, wsb, st); });
}

int bsa_forward_threshold_host(const bsa_params* p, float tau, const void* hQ, const void* hK,
                               const void* hV, void* hO, float* hlse, void* dQ, void* dK,
                               void* dV, void* dO, float* dlse, void* workspace,
                               size_t workspace_bytes, void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!std::isfinite(tau)) return BSA_ERR_INVALID;
  if (workspace_bytes <
      carve(threshold_shape(s), nullptr, nullptr) + bsa::attend_lists_scratch_bytes(s))
    return BSA_ERR_INVALID;
  return forward_host_pipelined(
      p, hQ, hK, hV, hO, hlse, dQ, dK, dV, dO, dlse, workspace, workspace_bytes, stream,
      [tau](const bsa_params* sub, void* q, void* k, void* v, void* o, float* l, void* ws,
            size_t wsb, void* st) {
        return bsa_forward_threshold(sub, tau, q, k, v, o, l, ws, wsb, st);
      });
}

int bsa_forward_extra_host(const bsa_params* p, int32_t n_extra, const void* hQ, const void* hK,
                           const void* hV, void* hO, float* hlse, void* dQ, void* dK, void* dV,
                           void* dO, float* dlse, void* workspace, size_t workspace_bytes,
                           void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (!extra_valid(s, n_extra)) return BSA_ERR_INVALID;
  if (workspace_bytes < carve(s, nullptr, nullptr) + extra_carve(s, n_extra, nullptr, nullptr))
    return BSA_ERR_INVALID;
  return forward_host_pipelined(
      p, hQ, hK, hV, hO, hlse, dQ, dK, dV, dO, dlse, workspace, workspace_bytes, stream,
      [n_extra](const bsa_params* sub, void* q, void* k, void* v, void* o, float* l, void* ws,
                size_t wsb, void* st) {
        return bsa_forward_extra(sub, n_extra, q, k, v, o, l, ws, wsb, st);
      },
      // 8 chunks: the token selection has a CTA per 128 query blocks, so a
      // chunk of few heads leaves most SMs idle (measured at 768p-5s: 35.3 ms
      // per call with 8 chunks, 44.2 with 14)
      8);
}

int bsa_forward_reblock_host(const bsa_params* p, const void* hQ, const void* hK,
                             const void* hV, void* hO, float* hlse, void* dQ, void* dK, void* dV,
                             void* dO, float* dlse, void* workspace, size_t workspace_bytes,
                             void* stream) {
  Shape s;
  int rc = shape_of(p, &s);
  if (rc) return rc;
  if (workspace_bytes < reblock_forward_carve(s, nullptr, nullptr)) return BSA_ERR_INVALID;
  return forward_host_pipelined(
      p, hQ, hK, hV, hO, hlse, dQ, dK, dV, dO, dlse, workspace, workspace_bytes, stream,
      [](const bsa_params* sub, void* q, void* k, void* v, void* o, float* l, void* ws,
         size_t wsb, void* st) { return bsa_forward_reblock(sub, q, k, v, o, l, ws, wsb, st); });
}

const char* bsa_status_string(int status) {
  switch (status) {
    case BSA_OK: return "ok";
    case BSA_ERR_INVALID: return "invalid argument";
    case BSA_ERR_ALIGN: return "pointer not 16-byte aligned";
    case BSA_ERR_CUDA: return "CUDA error";
    case BSA_ERR_TIMEOUT: return "bounded device wait expired";
    case BSA_ERR_UNSUPPORTED: return "unsupported device (needs sm_100) or driver";
    case BSA_ERR_SCRATCH: return "problem exceeds the static scratch of bsa_forward_noalloc";
    default: return "unknown status";
  }
}

int bsa_debug_expired_wait(int32_t* dev_status, uint64_t timeout_ns, void* stream) {
  if (!dev_status || !aligned(dev_status, 4)) return BSA_ERR_INVALID;
  if (timeout_ns > 10000000000ull) return BSA_ERR_INVALID;
  int rc = check_device();
  if (rc) return rc;
  return cuda_status(bsa::launch_expired_wait(dev_status, timeout_ns,
                                              static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
