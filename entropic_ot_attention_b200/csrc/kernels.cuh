// Kernel launchers shared between the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace eot {

// Kinds of per-position vector preparation (forward output and backward sweeps, §2.2).
enum PassKind { kPassOut = 0, kPassC1, kPassR2, kPassCk, kPassRk, kPassRF, kPassCF };

struct BwdVecArgs {
    int kind, k, R, H, BH, L, D;
    const float* logm;      // [B, L]
    const float* u_tail;    // [BH, R+1, L]
    const float* v_tail;    // [BH, R+1, L]
    const float* alpha;     // [R+1][BH*L]
    const float* beta;      // [R+1][BH*L]
    float *pr, *pc, *pcm2, *f, *hv, *m;
    float *xr, *yc;         // [2R][BH*L]
    // kPassR2 of the split alpha_R sweep: sadd = sum of the s1slots partial sums in s1part
    // (slot stride s1stride), the Pt dP row sums the column sweep beta_R left there
    const float* s1part;
    int s1slots;
    size_t s1stride;
    float* sadd;
    // kPassRF / kPassCF with at most kMaxFoldMods modifiers: also the operand rows of the folded
    // modifier product, 16 bf16 per position; modifier k takes entries 3k .. 3k + 2 as
    // xext = (-x_hi, -x_hi, -x_lo), yext = (y_hi, y_lo, y_hi) with x = x_hi + x_lo, y = y_hi + y_lo
    // (bf16 parts), so <xext_r, yext_c> = -sum_k xr_k[r] yc_k[c] up to the lo x lo products.
    __nv_bfloat16* xext;
    __nv_bfloat16* yext;
    // band-sum passes (kPassR2, kPassCk, kPassRk) of wide d = 128 bands: the column-bias operand
    // row of pcm2 for every position (band_ext_row with 1 / (scale log2 e) = isl2), or nullptr
    __nv_bfloat16* cext;
    float isl2;
};

// Log marginals of every batch row from the mask (and clears the status word); when given, also
// the tile bits of launch_tile_bits and the zero potential's masked log2 bias of launch_init_bias2
// ([BH, L]), in the same launch.
cudaError_t launch_prep_marginals(const Geom& g, const uint8_t* mask, int dustbin, float mass, float* logm,
                                  uint32_t* status, cudaStream_t st, uint32_t* bits = nullptr,
                                  float* bias2 = nullptr);
cudaError_t launch_dustbin_dots(const Geom& g, const void* P, const void* Qm, float s1, float* term, float* dense,
                                cudaStream_t st);
cudaError_t launch_simt_lse(const LsePass& p, cudaStream_t st);
// Every half-step of a forward without a dustbin on CUDA cores in one cooperative launch (row
// half-step template `row`; slots as in FusedSteps; gbar: 2 (T + R) zeroed counters).
cudaError_t launch_simt_lse_fused(const LsePass& row, const void* Q, const void* K, float* u_tail, float* v_tail,
                                  float* ub2, float* vb2, int T, int R, uint32_t* gbar, cudaStream_t st);
// The whole forward solve (every half-step, no dustbin) of each unit in one CTA, with the
// unit's band scores formed once into shared memory; when they fit (simt_resident_possible).
bool simt_resident_possible(const Geom& g);
cudaError_t launch_simt_resident(const LsePass& row, const void* Q, const void* K, float* u_tail, float* v_tail, int T,
                                 int R, cudaStream_t st);
cudaError_t launch_simt_bwd(const BwdPass& p, cudaStream_t st);
cudaError_t launch_bwd_vectors(const BwdVecArgs& a, cudaStream_t st);
// bias2 = log2(e) * pot over the active positions (pot null: a zero potential), -inf elsewhere
cudaError_t launch_init_bias2(const Geom& g, const float* logm, float* bias2, cudaStream_t st,
                              const float* pot = nullptr);
cudaError_t launch_tile_bits(const Geom& g, const float* logm, uint32_t* bits, cudaStream_t st);
cudaError_t launch_sq_norms(const void* a, const void* b, size_t n, int dtype, double* out, int n_sm,
                            cudaStream_t st);

// Projective contraction certificate: per tile pair wholly inside the band, tanh(Delta / 4) of
// exp(S) on the block's active real tokens (CUDA cores, scores in fp32).
struct ContractArgs {
    const void* Q;
    const void* K;
    const uint8_t* mask;   // [B, L] or null (every position real and active)
    int H, L, d;
    int nT;                // 128-position tiles, ceil(L / 128)
    int m;                 // offsets -m..m (m >= 0)
    int D;                 // dustbin index: positions >= D are left out; -1 without a dustbin
    float scale;
    float* kappa;          // [B H, nT, 2 m + 1]
};
cudaError_t launch_contraction(const ContractArgs& a, int dtype, int BH, cudaStream_t st);
cudaError_t launch_dustbin_lse(const LsePass& p, cudaStream_t st);
// (max, sum) partial of the dense dustbin row over the columns [lo, hi) (a part of a sequence)
cudaError_t launch_dustbin_part(const LsePass& p, int lo, int hi, float* part, cudaStream_t st);
cudaError_t launch_dustbin_bwd(const BwdPass& p, cudaStream_t st);

// Tensor-core (tcgen05 + TMA) kernels; return cudaErrorNotSupported when not built.
bool tc_supported(const Geom& g);
// 2-D TMA descriptor over a [rows, d] bf16 matrix, boxes of 64 elements x box_rows, 128-byte swizzle.
bool tma_map_bf16(CUtensorMap* m, const void* base, uint64_t rows, int d, int box_rows);
int sm_count();
cudaError_t launch_tc_lse(const LsePass& p, cudaStream_t st);
// Shifted half-steps hs0 .. hs0 + nhs - 1 of the forward schedule (even hs: row, odd: column;
// iteration hs / 2 writes slot 0 for the first T iterations and slot hs / 2 - T + 1 after) in one
// cooperative launch with grid-wide barriers (gbar[hs]: zeroed counters).  No dustbin.
struct FusedSteps {
    int hs0, nhs, T;
    float *u_tail, *v_tail, *ub2, *vb2;
    uint32_t* gbar;
    // d = 128: the column-bias operand rows of u and v ([BH L, 16] bf16; the first half-step
    // before this launch writes those of u)
    __nv_bfloat16 *ue, *ve;
    // the CTAs' item ranges (launch_schedule), or null for equal ranges
    const int* bounds;
};
cudaError_t launch_tc_lse_fused(const LsePass& row, const FusedSteps& f, cudaStream_t st);
// From the tile bits, in one launch: item ranges of equal weight for the band kernel's CTAs
// (bounds [kMaxBandCtas + 1]) and the order of the sweep kernel's row-tile jobs (jobs
// [BH L / 128]: those whose row tile holds an active token first, then the others, each in their
// natural order); every band and sweep launch of the problem's geometry can then take them.
cudaError_t launch_schedule(const Geom& g, const uint32_t* tile_bits, int* bounds, int* jobs, cudaStream_t st);
cudaError_t launch_tc_bwd(const BwdPass& p, cudaStream_t st);

// Staircase sweeps from the cached reference plan (cache.cu): out = f hv sum P m over the band, by
// rows (P a_r Pt) or by columns; P is the bf16 tile-relative band store written by the alpha_R row
// sweep (pcache).  Tensor-core bf16 problems without a dustbin and with h a multiple of 128.
struct CachedSweep {
    int H, L, h, BH, cpitch;
    const float* logm;
    const uint32_t* tile_bits;
    const __nv_bfloat16* P;
    const float* f;
    const float* hv;
    const float* m;
    float* out;
    uint32_t* status;
};
bool cached_sweeps_supported(const Geom& g);
cudaError_t launch_cached_sweep(const CachedSweep& a, bool column, cudaStream_t st);

// Forward iterations 1 .. T + R with one exponential per band entry per iteration (row sums and
// the plan entries of a 128-row strip on chip, column sums on the tensor core from the stored
// entries).  Iteration 1 starts from the row potential already in u_tail slot 0 (any finite row
// stabiliser, normally the first row half-step) and v = 0 in vb2.  No dustbin; T >= 1.
struct IterLaunch {
    Geom g;
    const void* Q;
    const void* K;
    const float* logm;
    const uint32_t* tile_bits;
    float* u_tail;
    float* v_tail;
    size_t pstride;           // (R + 1) L
    float* vb2;               // [BH, L] masked log2 v (initialised to v = 0)
    float* part;              // column partial sums (workspace region ``part``)
    uint32_t* gbar;           // 2 (T + R) zeroed grid-barrier counters
    uint32_t* status;
    int T, R;
    int fused;                // 0: one launch per iteration; 1: one cooperative launch, per-iteration
                              // launches if the device refuses it; 2: the cooperative launch only
};
// 0 when the problem does not fit the kernel, else 1 (one CTA per strip) or 2 (a CTA pair).
int iter_split(const Geom& g);
// *launched: kernels enqueued (1 cooperative launch, or 2 per iteration).
cudaError_t launch_tc_iter(const IterLaunch& p, cudaStream_t st, int* launched);

}  // namespace eot
