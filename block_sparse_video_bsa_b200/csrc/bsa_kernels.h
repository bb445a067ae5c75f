// Host-side launchers of the kernels (internal to libbsa.so).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>

namespace bsa {

// Runs `set` (a kernel-attribute setter) on the current device unless an
// earlier call on that device already succeeded.  The flags are atomics, so
// two host threads making their first call at the same time do not race; at
// worst both run `set`, which is idempotent.
template <class F>
cudaError_t once_per_device(std::atomic<bool> (&done)[64], F set) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return set();
  if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = set();
  if (e == cudaSuccess) done[dev].store(true, std::memory_order_release);
  return e;
}

struct Shape {
  int B, H, N;      // D is fixed at 128
  int nb;           // ceil(N / 128)
  int pb;           // prefix blocks
  int nbv;          // nb - pb
  int k_eff;        // min(top_k, nbv)
  int kcap;         // idx row length
  int variant;      // 0 anchor, 1 mean
  int prefix;       // prefix tokens
  int* dev_status;  // optional
};

// perm / Qp (optional): pool the permuted layout (row i of a head is Q row
// perm[i] of that head), writing the permuted rows to Qp.
cudaError_t launch_pool(const Shape& s, const void* Q, float* qpool, float* anchor,
                        cudaStream_t st, const int32_t* perm = nullptr, void* Qp = nullptr);
// kstat / vstat / lse_blk (optional, all or none): fp32 k~ and v~ (anchor
// variant) or mean k and mean v (mean variant), [B,H,nb,128], and the block
// LSE at the anchor (ln n for the mean variant), [B,H,nb].  perm / Kp / Vp
// (optional): summarize the permuted layout, writing its K and V rows.
cudaError_t launch_summarize(const Shape& s, const void* K, const void* V, const float* anchor,
                             float* kpool, void* ksum, void* vsum, float* bias, cudaStream_t st,
                             float* kstat = nullptr, float* vstat = nullptr,
                             float* lse_blk = nullptr, const int32_t* perm = nullptr,
                             void* Kp = nullptr, void* Vp = nullptr);
// Selection.  With `maps` (fp32 qpool / kpool as [BH, nb, 128] with 128-byte
// swizzle, boxes {32, select_tc_rows(s), 1} and {32, 128, 1}) and
// select_tc_rows(s) > 0 (rows of up to 3072 video blocks) the scores come
// from the tensor cores; otherwise (maps NULL, or longer rows) from the SIMT
// kernel.
int select_tc_rows(const Shape& s);
struct SelectMaps {
  CUtensorMap q, k;
};
cudaError_t launch_select(const Shape& s, const SelectMaps* maps, const float* qpool,
                          const float* kpool, int32_t* idx, int32_t* cnt, cudaStream_t st);
// Threshold selection: idx rows of length nb (kcap ignored), cnt per row.
cudaError_t launch_select_threshold(const Shape& s, float tau, const SelectMaps* maps,
                                    const float* qpool, const float* kpool, int32_t* idx,
                                    int32_t* cnt, cudaStream_t st);

struct AttendMaps {
  CUtensorMap q, k, v, ks, vs;   // bf16, box {64, 128, 1}, 128B swizzle
};
cudaError_t launch_attend(const Shape& s, const AttendMaps& maps, const int32_t* idx,
                          const int32_t* cnt, const float* bias, void* O, float* lse,
                          cudaStream_t st);
// Variable-length lists (row stride kcap, length cnt per row); `scratch`
// holds the schedule (attend_lists_scratch_bytes).
size_t attend_lists_scratch_bytes(const Shape& s);
cudaError_t launch_attend_lists(const Shape& s, const AttendMaps& maps, const int32_t* idx,
                                int kcap, const int32_t* cnt, const float* bias, void* O,
                                float* lse, void* scratch, cudaStream_t st);
// Extra tokens: K and V as 2-D [B*H*N, 128] bf16 with a {64, 1} box (row
// gathers), the side summary rows k~', v~' as [B*H, nb*scap, 128] with the
// usual {64, 128, 1} box.
struct AttendExtraMaps {
  CUtensorMap k2, v2, sk, sv;
};
cudaError_t launch_attend_extra(const Shape& s, const AttendMaps& maps,
                                const AttendExtraMaps& xmaps, const int32_t* idx,
                                const int32_t* extra, const int32_t* ecnt, int ecap,
                                const float* bias, const float* side_bias, const int32_t* side_cnt,
                                int scap, void* O, float* lse, cudaStream_t st);
// FP8 (e4m3) operands (layouts as bsa_fp8_operands in include/bsa.h).
struct Fp8Operands {
  void* q8;
  float* q_scale;
  void* k8;
  float* k_scale;
  void* vt8;
  float* v_scale;
  void* ks8;
  float* ks_scale;
  void* vst8;
  float* vs_scale;
  float* v_ref;
};
cudaError_t launch_quantize_fp8(const Shape& s, const void* Q, const void* K, const void* V,
                                const void* ksum, const void* vsum, const Fp8Operands& f,
                                cudaStream_t st);

struct AttendMapsFp8 {
  // uint8, box {128, 128, 1}, 128B swizzle: q8, k8 [BH, N, 128]; vt8
  // [BH, nb * 128, 128]; ks8 [BH, nb, 128]; vst8 [BH, ntile * 128, 128]
  CUtensorMap q, k, vt, ks, vst;
};
cudaError_t launch_attend_fp8(const Shape& s, const AttendMapsFp8& maps, const Fp8Operands& f,
                              const int32_t* idx, const float* bias, void* O, float* lse,
                              cudaStream_t st);

// Adaptive reblocking (reblock.cu).  Tree shape of one call (depends on
// N - prefix only): levels, chunk counts per level, partial-buffer slots.
struct ReblockPlan {
  int nv;                 // video tokens N - prefix
  int levels;             // ceil(log2(ceil(nv / 128)))
  int moment_chunks;      // 2048-row chunks of the key second moment
  int max_partials;       // chunk partials per head (largest level)
  int max_chunks[16];     // 2048-row chunks of the largest group, per level
  int max_pchunks[16];    // 512-position projection chunks of the largest group
                          // (0: every group is projected in its Gram CTA)
  int largest[16];        // tokens of the largest group, per level
};
ReblockPlan reblock_plan(const Shape& s);
struct ReblockBuffers {
  int32_t* perm_tmp;      // [BH, N]
  float* part;            // [BH, max_partials, 128, 128]
  float* psum;            // [BH, max_partials, 128]
  float* vdir;            // [BH, 2^levels, 128]
  float* moment;          // [BH, 128, 128] key second moment
  __nv_bfloat16* r_hi;    // [BH, 128, 128]
  __nv_bfloat16* r_lo;    // [BH, 128, 128]
  __nv_bfloat16* u;       // [BH, nv, 128]
  uint32_t* keys;         // [BH, nv]
};
struct ReblockMaps {
  CUtensorMap q, r_hi, r_lo;   // bf16, box {64, 128, 1}, 128B swizzle
  CUtensorMap u;               // the whitened rows [BH, nv, 128], same box (TMA stores)
};
cudaError_t launch_reblock(const Shape& s, const ReblockPlan& plan, const void* Q, const void* K,
                           const ReblockMaps& maps, const ReblockBuffers& w, int32_t* perm_out,
                           cudaStream_t st);
cudaError_t launch_permute_rows(const Shape& s, const void* Q, const void* K, const void* V,
                                const int32_t* perm, void* Qp, void* Kp, void* Vp,
                                cudaStream_t st);
cudaError_t launch_unpermute_rows(const Shape& s, const void* Op, const float* lsep,
                                  const int32_t* perm, void* O, float* lse, cudaStream_t st);

// Extra tokens (extra.cu).  Candidate-buffer capacity per query block,
// scratch of the selection, row capacity of the side summary table.
int extra_cand_cap(int n_extra);
size_t select_extra_scratch_bytes(const Shape& s, int n_extra);
int extra_side_cap(const Shape& s, int n_extra);
// tm_k: K as for the attention ([B*H, N, 128], box {64, 128, 1}, SW128).
cudaError_t launch_select_extra(const Shape& s, int n_extra, const CUtensorMap& tm_k,
                                const float* qpool, const int32_t* idx, int kcap,
                                const int32_t* cnt, int32_t* extra, int32_t* ecnt, void* scratch,
                                cudaStream_t st);
cudaError_t launch_extra_summaries(const Shape& s, int n_extra, const void* K, const void* V,
                                   const float* anchor, const float* kpool, const float* kstat,
                                   const float* vstat, const float* lse_blk, const int32_t* extra,
                                   const int32_t* ecnt, void* side_k, void* side_v,
                                   float* side_bias, int32_t* side_blk, int32_t* side_cnt,
                                   cudaStream_t st);

cudaError_t launch_expired_wait(int32_t* dev_status, uint64_t timeout_ns, cudaStream_t st);

}  // namespace bsa
