// gs_internal.h -- launchers shared between the kernel files and the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "gs_device.cuh"

namespace gsb {

// Digits of a least-significant-digit radix sort: pass i orders by
// (key >> shift[i]) & (2^bits[i] - 1).
struct RadixPlan {
  int passes = 0;
  int shift[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  int bits[8] = {0, 0, 0, 0, 0, 0, 0, 0};
};

// `key_bits` significant bits in the fewest passes of at most 8 bits; with
// `balanced` the bits are split evenly (13 -> 7 + 6), else 8 per pass.
RadixPlan make_radix_plan(int key_bits, bool balanced);
// Whether a plan's pair passes run single-sweep (the 64-bit keys of full-64
// mode; the 32-bit keys of the other paths take reduce-then-scan passes).
bool pair_passes_single_sweep(const RadixPlan& pairs, int sort_mode);

struct BinSortArgs {
  const float* bins;    // [n_views][n][4] binning records
  int n;
  int n_views;
  int mode;
  Grid grid;
  int64_t capacity;
  bool tile_emit;      // presort mode: pairs placed straight at their positions
  int gsize;           // tile emission: Gaussians per block
  int tile_bpv;        // tile emission: blocks per view
  bool column_emit;    // presort mode: emission ordered by tile column
  int cbits;           // column bits of a column-emission key (row << cbits | column)
  RadixPlan pairs;     // radix passes over the pair keys
  RadixPlan presort;   // radix passes over the per-Gaussian depth keys
  int emit_buf;        // which key/value buffer the emission writes
  uint64_t* keys[2];   // pair keys (64-bit, or 32-bit in presort mode)
  uint32_t* vals[2];   // pair ids; the final one is the caller's ids array
  uint64_t* pkeys[2];  // presort keys
  uint32_t* pvals[2];  // presort values
  uint32_t* totals;                  // [256] keys per digit of the current pass
  uint32_t* counts;                  // [256][counts_stride] radix digit counts / offsets
  int64_t counts_stride;             // partitions of the largest pass, a multiple of 4
  uint64_t* emit_lookback;           // [emit blocks]
  uint32_t* digit_hist;              // [8][256] digit counts of every single-sweep pass
  uint64_t* sweep_lookback;          // [partitions][256] single-sweep look-back words
  uint32_t* counters;                // [16] dynamic block counters
  uint32_t* status;
  WaitCfg wait;                      // emission look-back wait limit (and test stall)
  WaitCfg sort_wait;                 // single-sweep look-back wait limit (and test stall)
  int64_t* n_pairs;
  int64_t* n_items_dev;
  unsigned long long* pair_total;  // column emission: exact pair count
  uint4* crect;                      // tile / column emission: presorted rectangles [n_views * n]
  uint32_t* n_visible;               // [GS_MAX_VIEWS] visible Gaussians per view
  uint32_t* tile_totals;             // tile emission: pairs per tile [n_tiles]
  uint32_t* tile_base;               // tile emission: first position of each tile [n_tiles]
  int64_t* scan_n;                   // tile emission: blocks per view, for the scan
  bool count_ranges;                 // column emission: ranges from the tile counts
  int row_key_bytes;                 // column emission: 1, 2 (rows alone) or 4 bytes per key
  int* tile_diff;                    // count_ranges: [n_views][tiles_y + 1][tiles_x + 1]
  unsigned long long* view_pairs;    // count_ranges: pairs per view [GS_MAX_VIEWS]
  int64_t* ranges;
  int64_t n_tiles;     // n_views * tiles per view
};

// Quantised SH as the kernels read it: the codes of value j of Gaussian i at
// j * n_pad + i (planar, 8 or 16 bits) or in word 32 + ... of block
// (j, i / 32) of the packed layout; bounds (min, max) per (j, i / 256).
enum { kShqPlanar8 = 0, kShqPlanar16 = 1, kShqPacked = 2 };
struct ShQuant {
  const void* codes;
  const float2* bounds;
  int64_t n_pad;
  int64_t n_groups;
  float qmax;
  int kind;
};
inline ShQuant shq_of(const gs_sh_quant* q) {
  ShQuant r{};
  if (!q) return r;
  r.codes = q->codes;
  r.bounds = reinterpret_cast<const float2*>(q->bounds);
  r.n_pad = (q->n + GS_QUANT_GROUP - 1) / GS_QUANT_GROUP * GS_QUANT_GROUP;
  r.n_groups = r.n_pad / GS_QUANT_GROUP;
  r.qmax = (float)((1 << q->bits) - 1);
  r.kind = q->layout == GS_QUANT_PACKED ? kShqPacked : (q->bits == 8 ? kShqPlanar8 : kShqPlanar16);
  return r;
}

// The training step's tail fused into the projection backward: parameters
// (updated in place), both Adam moments, per-group learning rates (means,
// log-scales, quaternions, opacity logits, SH), the bias corrections, and the
// densification statistics (null accumulators: none).
struct AdamTail {
  float4 *p_means, *p_log_scales, *p_quats;
  float *p_logit, *p_sh;
  float4 *m_means, *m_log_scales, *m_quats;
  float *m_logit, *m_sh;
  float4 *v_means, *v_log_scales, *v_quats;
  float *v_logit, *v_sh;
  float lr[5];
  float b1, b2, eps, ibc1, ibc2;
  float* accum_plain;
  float* accum_abs;
  int* denom;
};

cudaError_t launch_project(const gs_params& p, const CamSet& cams, int n_views, float* records,
                           float* bins, int* radii, uint32_t* status, const WaitCfg& wc,
                           cudaStream_t stream);
cudaError_t launch_project_bwd(const gs_params& p, const CamSet& cams, int n_views,
                               const float* grad2d, const int* radii, const gs_grads& g,
                               cudaStream_t stream);
cudaError_t launch_project_bwd_adam(const gs_params& p, const CamSet& cams, int n_views,
                                    const float* grad2d, const int* radii, const AdamTail& t,
                                    cudaStream_t stream);
cudaError_t launch_bin_sort(const BinSortArgs& a, cudaStream_t stream);
cudaError_t launch_raster_fwd(const float* records, const uint32_t* ids, const int64_t* ranges,
                              int64_t capacity, const Grid& g, int n_views, int n,
                              const float bg[3], float* image,
                              float* final_T, uint32_t* n_contrib, uint8_t* warp_masks,
                              uint32_t* status, const WaitCfg& wc, cudaStream_t stream);
cudaError_t launch_raster_bwd(const float* records, const uint32_t* ids, const int64_t* ranges,
                              int64_t capacity, const Grid& g, int n_views, int n,
                              const float bg[3],
                              const float* dL_dimage, const float* final_T,
                              const uint32_t* n_contrib, const uint8_t* warp_masks,
                              float* grad2d, uint32_t* status, const WaitCfg& wc,
                              cudaStream_t stream);
cudaError_t launch_densify(const float* grad2d, const int* radii, int n_views, int n,
                           float* accum_plain, float* accum_abs, int* denom, cudaStream_t stream);
cudaError_t launch_adam(const gs_adam_group* groups, int n_groups, float b1, float b2, float eps,
                        int64_t step, cudaStream_t stream);

int64_t pair_partitions(int64_t items);     // radix partitions over pair keys
int64_t presort_partitions(int64_t items);  // radix partitions over depth keys
int64_t column_blocks(int64_t items);       // column-emission blocks
bool column_emission(const Grid& g);        // presort mode emits by column on this grid
bool tile_emission(const Grid& g);          // presort mode places pairs directly on this grid
bool count_ranges_fit(const Grid& g);       // a view's tile-count difference array fits a block
int tile_gsize(int64_t n);                  // tile emission: Gaussians per block
int64_t emit_blocks(int64_t items);

// densify_and_prune (densify.cu)
struct DensifyArgs {
  float grad_threshold;     // densify when accum > grad_threshold * denom, denom > 0
  float log_scale_split;    // split when the largest log-scale exceeds this, else clone
  float logit_min_opacity;  // prune when the opacity logit is below this
  float log_max_scale;      // prune when the largest log-scale exceeds this
  float log_split_shrink;   // a child's log-scales are the parent's minus this
};
struct DpTensorPtrs {       // the five parameter-shaped arrays (params, moments)
  float* means;             // float4 [n]
  float* log_scales;        // float4 [n]
  float* quats;             // float4 [n]
  float* logit;             // [n]
  float* sh;                // [n][K][3]
};
int64_t densify_blocks(int64_t n);
cudaError_t launch_densify_and_prune(const DpTensorPtrs& p_in, const DpTensorPtrs& m_in,
                                     const DpTensorPtrs& v_in, const float* accum,
                                     const int32_t* denom, const float* z, int n, int k3,
                                     const DensifyArgs& args, int8_t* codes,
                                     uint32_t* block_counts, int64_t capacity, int64_t* n_out,
                                     uint32_t* status, const DpTensorPtrs& p_out,
                                     const DpTensorPtrs& m_out, const DpTensorPtrs& v_out,
                                     cudaStream_t stream);

// Fused L1 + D-SSIM loss over [n_views][3][H][W] planes; `sums` holds
// 2 * n_views doubles followed by the block counter `done` (both cleared here).
size_t loss_smem_bytes();
cudaError_t launch_l1_dssim(const float* image, const float* target, int n_views, int H, int W,
                            float lambda, double* terms, float* grad, double* sums,
                            unsigned* done, cudaStream_t stream);

// Quantised SH state (gs_sh_quant, either layout; bounds [k3][n_pad / 256]).
cudaError_t launch_sh_quantize(const float* sh, const gs_sh_quant& q, cudaStream_t stream);
cudaError_t launch_sh_dequantize(const gs_sh_quant& q, float* sh, cudaStream_t stream);
cudaError_t launch_adam_sh_quant(const gs_sh_quant& q, const float* grad, uint16_t* m,
                                 uint16_t* v, float lr, float beta1, float beta2, float eps,
                                 int64_t step, int rounding, uint64_t seed, cudaStream_t stream);
// Output positions of densify_and_prune from its decisions: per-block output
// counts, their scan (checked against capacity, the count to *n_out), and the
// map src[o] = input of output o, bit 31 set where its moments start at zero.
cudaError_t launch_densify_map(const int8_t* decisions, int n, uint32_t* block_counts,
                               int64_t capacity, int64_t* n_out, uint32_t* src,
                               uint32_t* status, cudaStream_t stream);
// densify_and_prune of quantised SH: output positions from the decisions
// (block counts, their scan, the output -> input map src [n_out], bit 31 set
// where the moments start at zero), then every output group decoded from its
// inputs and encoded anew.
cudaError_t launch_densify_sh_quant(const gs_sh_quant& in, const uint16_t* m_in,
                                    const uint16_t* v_in, const int8_t* decisions,
                                    const gs_sh_quant& out, uint16_t* m_out, uint16_t* v_out,
                                    uint32_t* block_counts, int64_t* n_out_dev, uint32_t* src,
                                    uint32_t* status, cudaStream_t stream);

}  // namespace gsb
