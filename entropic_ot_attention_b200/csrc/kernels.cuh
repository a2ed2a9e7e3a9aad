// Kernel launchers shared between the C-ABI layer (api.cu) and the kernel files.
#pragma once

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
};

cudaError_t launch_prep_marginals(const Geom& g, const uint8_t* mask, int dustbin, float mass, float* logm,
                                  uint32_t* status, cudaStream_t st);
cudaError_t launch_dustbin_dots(const Geom& g, const void* P, const void* Qm, float s1, float* term, float* dense,
                                cudaStream_t st);
cudaError_t launch_simt_lse(const LsePass& p, cudaStream_t st);
cudaError_t launch_simt_bwd(const BwdPass& p, cudaStream_t st);
cudaError_t launch_bwd_vectors(const BwdVecArgs& a, cudaStream_t st);
cudaError_t launch_init_bias2(const Geom& g, const float* logm, float* bias2, cudaStream_t st);
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
cudaError_t launch_dustbin_bwd(const BwdPass& p, cudaStream_t st);

// Tensor-core (tcgen05 + TMA) kernels; return cudaErrorNotSupported when not built.
bool tc_supported(const Geom& g);
cudaError_t launch_tc_lse(const LsePass& p, cudaStream_t st);
// Shifted half-steps hs0 .. hs0 + nhs - 1 of the forward schedule (even hs: row, odd: column;
// iteration hs / 2 writes slot 0 for the first T iterations and slot hs / 2 - T + 1 after) in one
// cooperative launch with grid-wide barriers (gbar[hs]: zeroed counters).  No dustbin.
struct FusedSteps {
    int hs0, nhs, T;
    float *u_tail, *v_tail, *ub2, *vb2;
    uint32_t* gbar;
};
cudaError_t launch_tc_lse_fused(const LsePass& row, const FusedSteps& f, cudaStream_t st);
cudaError_t launch_tc_bwd(const BwdPass& p, cudaStream_t st);

}  // namespace eot
