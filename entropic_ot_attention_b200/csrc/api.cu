// C-ABI entry points of libeot (declared in include/eot.h): validation, workspace layout,
// and the order of the band sweeps that make up the forward and backward passes.
//
// Method: "Blockwise Differentiable Sinkhorn Attention", technical summary (gist.science
// 2605.08123).  §2.1: T stopped balanced steps, then R tail steps, then O = diag(1/a) P V.
// §2.2: the exact tail adjoint is a chain of band sweeps over one reference plan P(R,R);
// every other staircase factor is P(R,R) times per-row / per-column orbit factors.
// §2.3: the dustbin token is one more active position linked to every real token.
#include <math.h>
#include <string.h>

#include <atomic>
#include <vector>

#include "kernels.cuh"

// NVTX ranges around the passes of a call (host-side enqueue ranges that a timeline profiler
// pairs with the kernels they launch), compiled in only with -DEOT_NVTX.
#ifdef EOT_NVTX
#include <nvtx3/nvToolsExt.h>
namespace {
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};
}  // namespace
#define EOT_CAT2(a, b) a##b
#define EOT_CAT(a, b) EOT_CAT2(a, b)
#define EOT_RANGE(name) NvtxRange EOT_CAT(eot_nvtx_, __LINE__)(name)
#else
#define EOT_RANGE(name) ((void)0)
#endif

using namespace eot;

namespace {

// ---------------------------------------------------------------------------------------
// Launch accounting and optional per-kind CUDA-event timing (benchmark support)
// ---------------------------------------------------------------------------------------
enum ProfKind { kProfLse = 0, kProfOut = 1, kProfBwd = 2, kProfAux = 3, kProfStair = 4, kProfKinds = 5 };

struct Profiler {
    bool on = false;
    std::vector<cudaEvent_t> ev[kProfKinds];   // start/stop pairs, reused across sessions
    size_t used[kProfKinds] = {};
    double ms[kProfKinds] = {};
    long long count[kProfKinds] = {};
};
Profiler g_prof;
std::atomic<long long> g_launches{0};

// Runs f (which enqueues `nkernels` kernels on st) and, while profiling, brackets it with
// a pair of CUDA events on the same stream.
template <typename F>
cudaError_t tracked(int kind, int nkernels, cudaStream_t st, F&& f) {
    g_launches += nkernels;
    if (!g_prof.on) return f();
    auto& ev = g_prof.ev[kind];
    const size_t i = g_prof.used[kind];
    if (ev.size() < i + 2) {
        cudaEvent_t a, b;
        if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) return cudaErrorMemoryAllocation;
        ev.push_back(a);
        ev.push_back(b);
    }
    cudaError_t e = cudaEventRecord(ev[i], st);
    if (e != cudaSuccess) return e;
    e = f();
    if (e != cudaSuccess) return e;
    e = cudaEventRecord(ev[i + 1], st);
    g_prof.used[kind] = i + 2;
    g_prof.count[kind] += 1;
    return e;
}

// Forward schedule (process-wide; benchmark and test support): 0 and 1 run the half-step
// schedule (measured faster on every workload), 2 the one-exponential-per-iteration kernel in one
// cooperative launch, 3 that kernel with one launch per iteration.
std::atomic<int> g_fwd_schedule{0};
// Backward schedule (process-wide; measurement support): 0 recomputes the reference plan in every
// sweep, 1 caches it (bf16 band store written by the alpha_R sweep) for the staircase sweeps.
std::atomic<int> g_bwd_schedule{0};

bool tensor_core_ok(const eot_problem& p) { return p.dtype == EOT_BF16 && (p.d == 64 || p.d == 128); }

int resolve_impl(const eot_problem& p) {
    if (p.impl == EOT_IMPL_SIMT) return EOT_IMPL_SIMT;
    Geom g{};
    g.d = p.d;
    g.dtype = p.dtype;
    g.L = p.L;
    g.h = p.W / 2;
    const bool tc = tensor_core_ok(p) && tc_supported(g);
    if (p.impl == EOT_IMPL_TCGEN05) return tc ? EOT_IMPL_TCGEN05 : -1;
    return tc ? EOT_IMPL_TCGEN05 : EOT_IMPL_SIMT;
}

eot_status validate(const eot_problem* p) {
    if (!p) return EOT_ERR_INVALID_ARGUMENT;
    if (p->B < 0 || p->H < 0 || p->L < 0) return EOT_ERR_INVALID_ARGUMENT;
    if (p->L % 128 != 0) return EOT_ERR_INVALID_ARGUMENT;
    if (p->d < 8 || p->d > 128 || p->d % 8 != 0) return EOT_ERR_INVALID_ARGUMENT;
    if (p->W < 0 || p->T < 0 || p->R < 0 || p->R > kMaxR) return EOT_ERR_INVALID_ARGUMENT;
    if (p->dtype != EOT_FP32 && p->dtype != EOT_BF16) return EOT_ERR_INVALID_ARGUMENT;
    if (!(p->scale >= 0.f) || !isfinite(p->scale)) return EOT_ERR_INVALID_ARGUMENT;
    if (p->dustbin != 0 && p->dustbin != 1) return EOT_ERR_INVALID_ARGUMENT;
    if (p->dustbin_self != 0 && p->dustbin_self != 1) return EOT_ERR_INVALID_ARGUMENT;
    if (p->dustbin) {
        if (p->dustbin_index < 0 || p->dustbin_index >= p->L) return EOT_ERR_INVALID_ARGUMENT;
        if (!(p->dustbin_mass >= 0.f && p->dustbin_mass < 1.f)) return EOT_ERR_INVALID_ARGUMENT;
    }
    if (p->impl < EOT_IMPL_AUTO || p->impl > EOT_IMPL_TCGEN05) return EOT_ERR_INVALID_ARGUMENT;
    if (int64_t(p->B) * p->H > 65535) return EOT_ERR_UNSUPPORTED;
    if (int64_t(p->B) * p->H * p->L * int64_t(p->d) >= (int64_t(1) << 40)) return EOT_ERR_UNSUPPORTED;
    if (int64_t(p->B) * p->H * p->L >= (int64_t(1) << 31)) return EOT_ERR_UNSUPPORTED;   // TMA row coordinate
    if (resolve_impl(*p) < 0) return EOT_ERR_UNSUPPORTED;
    return EOT_OK;
}

bool empty(const eot_problem& p) { return int64_t(p.B) * p.H * p.L == 0; }

Geom make_geom(const eot_problem& p) {
    Geom g{};
    g.B = p.B;
    g.H = p.H;
    g.BH = p.B * p.H;
    g.L = p.L;
    g.d = p.d;
    g.h = p.W / 2;
    g.D = p.dustbin ? p.dustbin_index : -1;
    g.dself = p.dustbin_self;
    g.scale = p.scale > 0.f ? p.scale : 1.0f / sqrtf(float(p.d));
    g.dtype = p.dtype;
    return g;
}

template <typename T> T* at(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<char*>(ws) + off); }

#define EOT_TRY(expr)                                  \
    do {                                               \
        cudaError_t e_ = (expr);                       \
        if (e_ != cudaSuccess) return EOT_ERR_CUDA;    \
    } while (0)

cudaError_t run_lse(int impl, const LsePass& lp, cudaStream_t st) {
    const int nk = lp.g.D >= 0 ? 2 : 1;
    return tracked(kProfLse, nk, st, [&] {
        return impl == EOT_IMPL_TCGEN05 ? launch_tc_lse(lp, st) : launch_simt_lse(lp, st);
    });
}

cudaError_t run_bwd(int impl, const BwdPass& bp, cudaStream_t st, int kind = kProfBwd) {
    const int nk = bp.g.D >= 0 ? 2 : 1;
    return tracked(kind, nk, st, [&] {
        return impl == EOT_IMPL_TCGEN05 ? launch_tc_bwd(bp, st) : launch_simt_bwd(bp, st);
    });
}

template <typename F>
cudaError_t aux(cudaStream_t st, F&& f) { return tracked(kProfAux, 1, st, f); }

}  // namespace

// Forward/backward bodies that take the workspace as an already-resolved device address.
// (Also used by entry points that supply their own scratch.)
namespace eot {

int backward_schedule() { return g_bwd_schedule.load(); }

eot_status validate_problem(const eot_problem* p) { return validate(p); }

eot_status forward_impl(const eot_problem* p, const void* Q, const void* K, const void* V, const uint8_t* mask,
                        void* O, float* u_tail, float* v_tail, void* ws, cudaStream_t st) {
    EOT_RANGE("eot forward");
    const Geom g = make_geom(*p);
    const int impl = resolve_impl(*p);
    const WsLayout w = ws_layout(*p, false);
    const size_t L = size_t(p->L), R = size_t(p->R);
    const size_t pstride = (R + 1) * L;
    uint32_t* status = at<uint32_t>(ws, w.status);
    float* logm = at<float>(ws, w.logm);
    float* sd_row = p->dustbin ? at<float>(ws, w.sd_row) : nullptr;
    float* sd_col = p->dustbin ? at<float>(ws, w.sd_col) : nullptr;
    float* ub2 = at<float>(ws, w.ub2);
    float* vb2 = at<float>(ws, w.vb2);
    uint32_t* tbits = at<uint32_t>(ws, w.tbits);

    // marginals, tile bits and the zero potential's masked log2 bias (v = 0) in one launch
    EOT_TRY(aux(st, [&] {
        return launch_prep_marginals(g, mask, p->dustbin, p->dustbin_mass, logm, status, st, tbits, vb2);
    }));
    float* dpart = p->dustbin ? at<float>(ws, w.dpart) : nullptr;
    uint32_t* dcnt = p->dustbin ? at<uint32_t>(ws, w.dcnt) : nullptr;
    if (p->dustbin) {
        EOT_TRY(cudaMemsetAsync(dcnt, 0, size_t(g.BH) * sizeof(uint32_t), st));
        EOT_TRY(aux(st, [&] { return launch_dustbin_dots(g, Q, K, g.scale, sd_row, sd_col, st); }));
    }
    const size_t tail_bytes = size_t(g.BH) * pstride * sizeof(float);
    EOT_TRY(cudaMemsetAsync(u_tail, 0, tail_bytes, st));
    EOT_TRY(cudaMemsetAsync(v_tail, 0, tail_bytes, st));

    LsePass row{};
    row.g = g;
    row.X = Q;
    row.Y = K;
    row.logm = logm;
    row.pstride = pstride;
    row.sd_term = sd_row;
    row.sd_dense = sd_col;
    row.dpart = dpart;
    row.dcnt = dcnt;
    row.status = status;
    row.tile_bits = tbits;
    int* bounds = at<int>(ws, w.bounds);
    int* jobs = nullptr;
    if (impl == EOT_IMPL_TCGEN05) {
        // every band launch of this call takes item ranges of equal weight, and the output sweep
        // its row-tile jobs active ones first
        jobs = at<int>(ws, w.jobs);
        EOT_TRY(aux(st, [&] { return launch_schedule(g, tbits, bounds, jobs, st); }));
        row.bounds = bounds;
    }
    row.colbias2 = vb2;
    row.out_bias2 = ub2;
    LsePass col = row;
    col.colbias2 = ub2;
    col.out_bias2 = vb2;
    col.X = K;
    col.Y = Q;
    col.sd_term = sd_col;
    col.sd_dense = sd_row;

    bool first = true;
    auto step = [&](int k_in, int k_out) -> cudaError_t {
        EOT_RANGE("eot iteration (row + column half-step)");
        // row half-step: u(k_out) from v(k_in); column half-step: v(k_out) from u(k_out)
        row.colpot = v_tail + size_t(k_in) * L;
        row.stab = first ? nullptr : u_tail + size_t(k_in) * L;
        row.out = u_tail + size_t(k_out) * L;
        cudaError_t e = run_lse(impl, row, st);
        if (e != cudaSuccess) return e;
        first = false;
        col.colpot = u_tail + size_t(k_out) * L;
        col.stab = v_tail + size_t(k_in) * L;
        col.out = v_tail + size_t(k_out) * L;
        return run_lse(impl, col, st);
    };
    // Tensor-core path: the first half-step (running maximum) on its own, then either every
    // iteration with one exponential per band entry (iter.cu, no dustbin: the first row
    // half-step's u is the row stabiliser of iteration 1, which recomputes it), or every later
    // half-step in one cooperative launch with grid-wide barriers between them (with a dustbin
    // that launch also sums each half-step's dense dustbin row).  If the device cannot hold the
    // whole grid at once the iterations / half-steps run as separate launches.
    const int n_half = 2 * (p->T + p->R);
    bool fused = false;
    const int sched = g_fwd_schedule.load();
    const bool use_iter = impl == EOT_IMPL_TCGEN05 && sched >= 2 && iter_schedule_possible(*p) && iter_split(g) > 0;
    if (sched >= 2 && !use_iter) return EOT_ERR_UNSUPPORTED;
    if (use_iter) {
        EOT_TRY(run_lse(impl, [&] {
            LsePass r0 = row;
            r0.colpot = v_tail;
            r0.stab = nullptr;
            r0.out = u_tail;
            return r0;
        }(), st));
        uint32_t* gbar = at<uint32_t>(ws, w.gbar);
        EOT_TRY(cudaMemsetAsync(gbar, 0, size_t(n_half) * sizeof(uint32_t), st));
        IterLaunch il{};
        il.g = g;
        il.Q = Q;
        il.K = K;
        il.logm = logm;
        il.tile_bits = tbits;
        il.u_tail = u_tail;
        il.v_tail = v_tail;
        il.pstride = pstride;
        il.vb2 = vb2;
        il.part = at<float>(ws, w.part);
        il.gbar = gbar;
        il.status = status;
        il.T = p->T;
        il.R = p->R;
        il.fused = sched == 2 ? 2 : sched == 3 ? 0 : 1;
        int launched = 0;
        EOT_TRY(tracked(kProfLse, 0, st, [&] { return launch_tc_iter(il, st, &launched); }));
        g_launches += launched;
    } else if (impl == EOT_IMPL_TCGEN05 && n_half >= 2) {
        // (the fused d = 128 half-steps of a band of W >= 512 take the column bias from these rows)
        const bool bext = w.bext && g.h >= 256;
        __nv_bfloat16* ue = bext ? at<__nv_bfloat16>(ws, w.ue) : nullptr;
        __nv_bfloat16* ve = bext ? at<__nv_bfloat16>(ws, w.ve) : nullptr;
        EOT_TRY(run_lse(impl, [&] {
            LsePass r0 = row;
            r0.colpot = v_tail;
            r0.stab = nullptr;
            r0.out = u_tail + (p->T > 0 ? 0 : L);
            r0.ext_out = ue;
            return r0;
        }(), st));
        uint32_t* gbar = at<uint32_t>(ws, w.gbar);
        EOT_TRY(cudaMemsetAsync(gbar, 0, size_t(n_half) * sizeof(uint32_t), st));
        FusedSteps f{1, n_half - 1, p->T, u_tail, v_tail, ub2, vb2, gbar, ue, ve, row.bounds};
        const cudaError_t e = tracked(kProfLse, 1, st, [&] { return launch_tc_lse_fused(row, f, st); });
        if (e == cudaSuccess) fused = true;
        else if (e == cudaErrorCooperativeLaunchTooLarge) {
            (void)cudaGetLastError();
            g_launches -= 1;   // the refused launch
        }
        else return EOT_ERR_CUDA;
        if (!fused) {
            // finish the first iteration's column half-step, then the rest one launch each
            first = false;
            const int k_out = p->T > 0 ? 0 : 1;
            col.colpot = u_tail + size_t(k_out) * L;
            col.stab = v_tail;
            col.out = v_tail + size_t(k_out) * L;
            EOT_TRY(run_lse(impl, col, st));
            for (int t = 1; t < p->T; ++t) EOT_TRY(step(0, 0));
            for (int k = (p->T > 0 ? 1 : 2); k <= p->R; ++k) EOT_TRY(step(k - 1, k));
        }
    } else if (impl != EOT_IMPL_TCGEN05 && n_half >= 2 && simt_resident_possible(g)) {
        // CUDA-core path, small units: the whole solve of each unit in one CTA, scores formed once
        EOT_TRY(tracked(kProfLse, 1, st, [&] { return launch_simt_resident(row, Q, K, u_tail, v_tail, p->T, p->R, st); }));
    } else if (impl != EOT_IMPL_TCGEN05 && g.D < 0 && n_half >= 2) {
        // CUDA-core path without a dustbin: every half-step in one cooperative launch (the kernel
        // keeps no running stabiliser, so the first half-step needs no separate launch).
        uint32_t* gbar = at<uint32_t>(ws, w.gbar);
        EOT_TRY(cudaMemsetAsync(gbar, 0, size_t(n_half) * sizeof(uint32_t), st));
        const cudaError_t e = tracked(kProfLse, 1, st, [&] {
            return launch_simt_lse_fused(row, Q, K, u_tail, v_tail, ub2, vb2, p->T, p->R, gbar, st);
        });
        if (e == cudaErrorCooperativeLaunchTooLarge) {
            (void)cudaGetLastError();
            g_launches -= 1;   // the refused launch
            for (int t = 0; t < p->T; ++t) EOT_TRY(step(0, 0));
            for (int k = 1; k <= p->R; ++k) EOT_TRY(step(k - 1, k));
        } else if (e != cudaSuccess) {
            return EOT_ERR_CUDA;
        }
    } else {
        for (int t = 0; t < p->T; ++t) EOT_TRY(step(0, 0));                 // stopped base
        for (int k = 1; k <= p->R; ++k) EOT_TRY(step(k - 1, k));            // differentiable tail
    }

    // Output O = diag(1/a) P(R,R) V (a vector sweep with coefficients P / a_r).
    EOT_RANGE("eot output sweep");
    BwdVecArgs va{};
    va.kind = kPassOut;
    va.R = p->R;
    va.H = g.H;
    va.BH = g.BH;
    va.L = g.L;
    va.logm = logm;
    va.u_tail = u_tail;
    va.v_tail = v_tail;
    va.D = g.D;
    va.pr = at<float>(ws, w.opr);
    va.pc = at<float>(ws, w.opc);
    va.pcm2 = at<float>(ws, w.opcm);
    va.f = va.hv = va.m = nullptr;            // unused by the output pass
    EOT_TRY(aux(st, [&] { return launch_bwd_vectors(va, st); }));
    BwdPass op{};
    op.g = g;
    op.X = Q;
    op.Y = K;
    op.Z = V;
    op.logm = logm;
    op.pr = va.pr;
    op.pc = va.pc;
    op.pcm2 = va.pcm2;
    op.vout = O;
    op.vscale = 1.f;
    op.v_dp = 0;
    op.nmod = 0;
    op.sd_term = sd_row;
    op.sd_dense = sd_col;
    op.dpart = dpart;
    op.dcnt = dcnt;
    op.status = status;
    op.tile_bits = tbits;
    op.jobs = jobs;
    EOT_TRY(run_bwd(impl, op, st, kProfOut));
    return EOT_OK;
}

// The output of given potentials (§2.1): O = diag(1/a) P V with P_ij = exp(S_ij + u_i + v_j) on the
// band and a_i = exp(log_marg_i) (no dustbin); the forward's output sweep with a one-slot tail.
eot_status output_impl(const eot_problem* p, const void* Q, const void* K, const void* V, const float* log_marg,
                       const float* u, const float* v, void* O, void* ws, cudaStream_t st) {
    EOT_RANGE("eot band output");
    const Geom g = make_geom(*p);
    const int impl = resolve_impl(*p);
    const WsLayout w = ws_layout(*p, false);
    uint32_t* status = at<uint32_t>(ws, w.status);
    EOT_TRY(cudaMemsetAsync(status, 0, sizeof(uint32_t), st));
    uint32_t* tbits = at<uint32_t>(ws, w.tbits);
    EOT_TRY(aux(st, [&] { return launch_tile_bits(g, log_marg, tbits, st); }));
    BwdVecArgs va{};
    va.kind = kPassOut;
    va.R = 0;
    va.H = g.H;
    va.BH = g.BH;
    va.L = g.L;
    va.logm = log_marg;
    va.u_tail = u;
    va.v_tail = v;
    va.D = g.D;
    va.pr = at<float>(ws, w.opr);
    va.pc = at<float>(ws, w.opc);
    va.pcm2 = at<float>(ws, w.opcm);
    va.f = va.hv = va.m = nullptr;
    EOT_TRY(aux(st, [&] { return launch_bwd_vectors(va, st); }));
    BwdPass op{};
    op.g = g;
    op.X = Q;
    op.Y = K;
    op.Z = V;
    op.logm = log_marg;
    op.pr = va.pr;
    op.pc = va.pc;
    op.pcm2 = va.pcm2;
    op.vout = O;
    op.vscale = 1.f;
    op.v_dp = 0;
    op.nmod = 0;
    op.status = status;
    op.tile_bits = tbits;
    EOT_TRY(run_bwd(impl, op, st, kProfOut));
    return EOT_OK;
}

// One half-step on its own (§2.1): out = log_marg - LSE over the band of (scale <x_i, y_j> + in_j),
// with a running maximum (the online form of the first half-step of a solve), so that any finite
// input potential is accepted.
// With a dustbin (own_lo <= own_hi, dust_part not null) every real row also takes the dustbin
// column term S_iD + in_D, and the dense dustbin row is returned as a (max, sum) partial over the
// columns [own_lo, own_hi) instead of a finished potential.
eot_status half_step_impl(const eot_problem* p, const void* X, const void* Y, const float* log_marg,
                          const float* in, float* out, void* ws, cudaStream_t st, int own_lo = 0,
                          int own_hi = 0, float* dust_part = nullptr) {
    EOT_RANGE("eot band half-step");
    const Geom g = make_geom(*p);
    const int impl = resolve_impl(*p);
    const WsLayout w = ws_layout(*p, false);
    uint32_t* status = at<uint32_t>(ws, w.status);
    EOT_TRY(cudaMemsetAsync(status, 0, sizeof(uint32_t), st));
    float* sd_row = nullptr;
    float* sd_col = nullptr;
    if (p->dustbin) {
        sd_row = at<float>(ws, w.sd_row);
        sd_col = at<float>(ws, w.sd_col);
        EOT_TRY(cudaMemsetAsync(at<uint32_t>(ws, w.dcnt), 0, size_t(g.BH) * sizeof(uint32_t), st));
        EOT_TRY(aux(st, [&] { return launch_dustbin_dots(g, X, Y, g.scale, sd_row, sd_col, st); }));
    }
    float* in_b2 = at<float>(ws, w.vb2);
    float* out_b2 = at<float>(ws, w.ub2);
    uint32_t* tbits = at<uint32_t>(ws, w.tbits);
    EOT_TRY(aux(st, [&] { return launch_init_bias2(g, log_marg, in_b2, st, in); }));
    EOT_TRY(aux(st, [&] { return launch_tile_bits(g, log_marg, tbits, st); }));
    LsePass lp{};
    lp.g = g;
    lp.X = X;
    lp.Y = Y;
    lp.logm = log_marg;
    lp.colpot = in;
    lp.stab = nullptr;
    lp.out = out;
    lp.pstride = size_t(p->L);
    lp.colbias2 = in_b2;
    lp.out_bias2 = out_b2;
    lp.tile_bits = tbits;
    lp.status = status;
    if (p->dustbin) {
        lp.sd_term = sd_row;
        lp.sd_dense = sd_col;
        lp.dpart = at<float>(ws, w.dpart);
        lp.dcnt = at<uint32_t>(ws, w.dcnt);
    }
    EOT_TRY(run_lse(impl, lp, st));
    if (p->dustbin) EOT_TRY(aux(st, [&] { return launch_dustbin_part(lp, own_lo, own_hi, dust_part, st); }));
    return EOT_OK;
}

eot_status backward_impl(const eot_problem* p, const void* Q, const void* K, const void* V, const uint8_t* mask,
                         const float* u_tail, const float* v_tail, const void* dO, void* dQ, void* dK, void* dV,
                         void* ws, cudaStream_t st) {
    EOT_RANGE("eot backward");
    const Geom g = make_geom(*p);
    const int impl = resolve_impl(*p);
    const WsLayout w = ws_layout(*p, true);
    const int R = p->R;
    const size_t vecn = align256(size_t(g.BH) * g.L * sizeof(float)) / sizeof(float);
    uint32_t* status = at<uint32_t>(ws, w.status);
    float* logm = at<float>(ws, w.logm);
    float *sd_row = nullptr, *sd_col = nullptr, *e1 = nullptr, *e2 = nullptr;
    uint32_t* tbits = at<uint32_t>(ws, w.tbits);
    // marginals and tile bits in one launch
    EOT_TRY(aux(st, [&] {
        return launch_prep_marginals(g, mask, p->dustbin, p->dustbin_mass, logm, status, st, tbits);
    }));
    float* dpart = p->dustbin ? at<float>(ws, w.dpart) : nullptr;
    uint32_t* dcnt = p->dustbin ? at<uint32_t>(ws, w.dcnt) : nullptr;
    if (p->dustbin) {
        EOT_TRY(cudaMemsetAsync(dcnt, 0, size_t(g.BH) * sizeof(uint32_t), st));
        sd_row = at<float>(ws, w.sd_row);
        sd_col = at<float>(ws, w.sd_col);
        e1 = at<float>(ws, w.e1);
        e2 = at<float>(ws, w.e2);
        EOT_TRY(aux(st, [&] { return launch_dustbin_dots(g, Q, K, g.scale, sd_row, sd_col, st); }));
        // e1[r] = <dO_r, V_D>, e2[r] = <dO_D, V_r>
        EOT_TRY(aux(st, [&] { return launch_dustbin_dots(g, dO, V, 1.f, e1, e2, st); }));
    }
    float* alpha = at<float>(ws, w.alpha);
    float* beta = at<float>(ws, w.beta);

    BwdVecArgs va{};
    va.R = R;
    va.H = g.H;
    va.BH = g.BH;
    va.L = g.L;
    va.logm = logm;
    va.u_tail = u_tail;
    va.v_tail = v_tail;
    va.alpha = alpha;
    va.beta = beta;
    va.D = g.D;
    va.pr = at<float>(ws, w.pr);
    va.pc = at<float>(ws, w.pc);
    va.pcm2 = at<float>(ws, w.pcm);
    va.f = at<float>(ws, w.f);
    va.hv = at<float>(ws, w.hv);
    va.m = at<float>(ws, w.m);
    va.xr = R > 0 ? at<float>(ws, w.xr) : nullptr;
    // band sums of a wide d = 128 band on the tensor cores take their column bias as operand rows
    __nv_bfloat16* cext = (impl == EOT_IMPL_TCGEN05 && w.bcext) ? at<__nv_bfloat16>(ws, w.cext) : nullptr;
    va.cext = cext;
    va.isl2 = float(1.0 / double(g.scale * kLog2e));
    va.yc = R > 0 ? at<float>(ws, w.yc) : nullptr;

    // Row orientation: S = Q K^T, dP = dO V^T.  Column orientation: S^T = K Q^T, dP^T = V dO^T.
    BwdPass rowp{};
    rowp.g = g;
    rowp.X = Q;
    rowp.Y = K;
    rowp.A = dO;
    rowp.Bm = V;
    rowp.logm = logm;
    rowp.pr = va.pr;
    rowp.pc = va.pc;
    rowp.pcm2 = va.pcm2;
    rowp.sd_term = sd_row;
    rowp.sd_dense = sd_col;
    rowp.dp_term = e1;
    rowp.dp_dense = e2;
    rowp.dpart = dpart;
    rowp.dcnt = dcnt;
    rowp.zero_vec = at<float>(ws, w.zero);
    rowp.status = status;
    rowp.tile_bits = tbits;
    if (impl == EOT_IMPL_TCGEN05) {
        int* bounds = at<int>(ws, w.bounds);
        int* jobs = at<int>(ws, w.jobs);
        EOT_TRY(aux(st, [&] { return launch_schedule(g, tbits, bounds, jobs, st); }));
        rowp.bounds = bounds;
        rowp.jobs = jobs;
    }
    EOT_TRY(cudaMemsetAsync(at<float>(ws, w.zero), 0, vecn * sizeof(float), st));
    BwdPass colp = rowp;
    colp.X = K;
    colp.Y = Q;
    colp.A = V;
    colp.Bm = dO;
    colp.sd_term = sd_col;
    colp.sd_dense = sd_row;
    colp.dp_term = e2;
    colp.dp_dense = e1;

    auto vec = [&](int kind, int k) -> cudaError_t {
        va.kind = kind;
        va.k = k;
        return aux(st, [&] { return launch_bwd_vectors(va, st); });
    };
    auto scalar_pass = [&](BwdPass bp, float* out, bool dp) -> cudaError_t {
        bp.sout = out;
        bp.f = va.f;
        bp.hv = va.hv;
        bp.m = va.m;
        bp.s_dp = dp ? 1 : 0;
        return run_bwd(impl, bp, st);
    };

    // With the split alpha_R sweep (tensor-core kernels), the column sweep C1 also leaves the
    // partial row sums of Pt dP in s1part, and alpha_R becomes a staircase-form band sum plus them.
    const bool split = R > 0 && impl == EOT_IMPL_TCGEN05 && w.s1split;
    float* s1part = split ? at<float>(ws, w.s1part) : nullptr;
    const int s1E = s1_reach(p->W);
    const int s1slots = int(s1_slots(p->W));
    if (split) EOT_TRY(cudaMemsetAsync(s1part, 0, size_t(s1slots) * vecn * sizeof(float), st));

    // C1: beta_R = colsum(P(R,R) * dP) and dV = P(R,R)^T (dO / a)   (one column sweep)
    EOT_TRY(vec(kPassC1, 0));
    {
        EOT_RANGE("eot backward: beta_R, dV");
        BwdPass bp = colp;
        if (R > 0) {
            bp.sout = beta + size_t(R) * vecn;
            bp.f = va.f;
            bp.hv = va.hv;
            bp.m = nullptr;
            bp.s_dp = 1;
            bp.s1part = s1part;
            bp.s1stride = vecn;
            bp.s1E = s1E;
        }
        bp.vout = dV;
        bp.Z = dO;
        bp.vscale = 1.f;
        bp.v_dp = 0;
        bp.nmod = 0;
        EOT_TRY(run_bwd(impl, bp, st));
    }
    if (R > 0) {
        // R2: alpha_R = rowsum(P(R,R) * dP) - P(R,R) (beta_R / b)
        EOT_RANGE("eot backward: staircase vectors");
        // With the cached schedule this sweep also stores its plan entries for the staircase.
        const bool cached = impl == EOT_IMPL_TCGEN05 && cache_plan_possible(*p) && cached_sweeps_supported(g);
        __nv_bfloat16* pcache = cached ? at<__nv_bfloat16>(ws, w.pcache) : nullptr;
        if (split) {
            va.s1part = s1part;
            va.s1slots = s1slots;
            va.s1stride = vecn;
            va.sadd = at<float>(ws, w.sadd);
        }
        EOT_TRY(vec(kPassR2, 0));
        va.s1part = nullptr;
        va.sadd = nullptr;
        if (split) {
            // alpha_R = (row sums of Pt dP from C1) + hv_r sum_c Pt_rc m_c: a staircase-form sum
            BwdPass bp = rowp;
            bp.sout = alpha + size_t(R) * vecn;
            bp.f = va.f;
            bp.hv = va.hv;
            bp.m = va.m;
            bp.s_dp = 0;
            bp.sadd = at<float>(ws, w.sadd);
            bp.cext = cext;
            EOT_TRY(run_bwd(impl, bp, st, kProfStair));
        } else {
            BwdPass bp = rowp;
            bp.pcache = pcache;
            EOT_TRY(scalar_pass(bp, alpha + size_t(R) * vecn, true));
        }
        CachedSweep cs{};
        cs.H = g.H;
        cs.L = g.L;
        cs.h = g.h;
        cs.BH = g.BH;
        cs.cpitch = 2 * g.h + 128;
        cs.logm = logm;
        cs.tile_bits = tbits;
        cs.P = pcache;
        cs.f = va.f;
        cs.hv = va.hv;
        cs.m = va.m;
        cs.status = status;
        for (int k = R - 1; k >= 1; --k) {
            // beta_k = -P(k+1,k)^T (alpha_{k+1} / a), alpha_k = -P(k,k) (beta_k / b)
            EOT_TRY(vec(kPassCk, k));
            if (cached) {
                cs.out = beta + size_t(k) * vecn;
                EOT_TRY(tracked(kProfStair, 1, st, [&] { return launch_cached_sweep(cs, true, st); }));
            } else {
                BwdPass bp = colp;
                bp.sout = beta + size_t(k) * vecn;
                bp.f = va.f;
                bp.hv = va.hv;
                bp.m = va.m;
                bp.s_dp = 0;
                bp.cext = cext;
                EOT_TRY(run_bwd(impl, bp, st, kProfStair));
            }
            EOT_TRY(vec(kPassRk, k));
            if (cached) {
                cs.out = alpha + size_t(k) * vecn;
                EOT_TRY(tracked(kProfStair, 1, st, [&] { return launch_cached_sweep(cs, false, st); }));
            } else {
                BwdPass bp = rowp;
                bp.sout = alpha + size_t(k) * vecn;
                bp.f = va.f;
                bp.hv = va.hv;
                bp.m = va.m;
                bp.s_dp = 0;
                bp.cext = cext;
                EOT_TRY(run_bwd(impl, bp, st, kProfStair));
            }
        }
    }
    // dQ = scale dS K (row sweep), dK = scale dS^T Q (column sweep); dS = P(R,R) (dP - sum x y^T).
    // Tensor-core problems without a dustbin take the modifier term out of the dP product.
    const bool fold = impl == EOT_IMPL_TCGEN05 && w.fold && 2 * R <= kMaxFoldMods;
    for (int orient = 0; orient < 2; ++orient) {
        EOT_RANGE(orient == 0 ? "eot backward: dQ" : "eot backward: dK");
        va.xext = fold ? at<__nv_bfloat16>(ws, w.xext) : nullptr;
        va.yext = fold ? at<__nv_bfloat16>(ws, w.yext) : nullptr;
        EOT_TRY(vec(orient == 0 ? kPassRF : kPassCF, 0));
        va.xext = va.yext = nullptr;
        BwdPass bp = orient == 0 ? rowp : colp;
        if (fold) {
            bp.xext = at<__nv_bfloat16>(ws, w.xext);
            bp.yext = at<__nv_bfloat16>(ws, w.yext);
        }
        bp.vout = orient == 0 ? dQ : dK;
        bp.Z = orient == 0 ? K : Q;
        bp.vscale = g.scale;
        bp.v_dp = 1;
        bp.nmod = 2 * R;
        for (int k = 0; k < 2 * R; ++k) {
            bp.xr[k] = va.xr + size_t(k) * vecn;
            bp.yc[k] = va.yc + size_t(k) * vecn;
        }
        EOT_TRY(run_bwd(impl, bp, st));
    }
    return EOT_OK;
}

}  // namespace eot

// ---------------------------------------------------------------------------------------
// Exported C ABI
// ---------------------------------------------------------------------------------------
extern "C" {

int eot_abi_version(void) { return EOT_ABI_VERSION; }

eot_status eot_validate(const eot_problem* p) { return validate(p); }

int eot_resolved_impl(const eot_problem* p) {
    if (validate(p) != EOT_OK) return -1;
    return resolve_impl(*p);
}

size_t eot_workspace_bytes(const eot_problem* p, int for_backward) {
    if (validate(p) != EOT_OK || empty(*p)) return 0;
    return ws_layout(*p, for_backward != 0).total;
}

const char* eot_status_string(eot_status s) {
    switch (s) {
        case EOT_OK: return "ok";
        case EOT_ERR_INVALID_ARGUMENT: return "invalid argument";
        case EOT_ERR_UNSUPPORTED: return "unsupported problem for this library";
        case EOT_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case EOT_ERR_CUDA: return "CUDA error";
        case EOT_ERR_NONFINITE: return "non-finite potential produced on the device";
        case EOT_ERR_TIMEOUT: return "a bounded device wait ran out";
    }
    return "unknown status";
}

eot_status eot_sinkhorn_fwd(const eot_problem* p, const void* Q, const void* K, const void* V, const uint8_t* mask,
                            void* O, float* u_tail, float* v_tail, void* workspace, size_t workspace_bytes,
                            void* stream) {
    eot_status s = validate(p);
    if (s != EOT_OK) return s;
    if (empty(*p)) return EOT_OK;
    if (!Q || !K || !V || !O || !u_tail || !v_tail || !workspace) return EOT_ERR_INVALID_ARGUMENT;
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return EOT_ERR_INVALID_ARGUMENT;
    if (workspace_bytes < ws_layout(*p, false).total) return EOT_ERR_WORKSPACE_TOO_SMALL;
    return forward_impl(p, Q, K, V, mask, O, u_tail, v_tail, workspace, static_cast<cudaStream_t>(stream));
}

eot_status eot_sinkhorn_bwd(const eot_problem* p, const void* Q, const void* K, const void* V, const uint8_t* mask,
                            const float* u_tail, const float* v_tail, const void* dO, void* dQ, void* dK, void* dV,
                            void* workspace, size_t workspace_bytes, void* stream) {
    eot_status s = validate(p);
    if (s != EOT_OK) return s;
    if (empty(*p)) return EOT_OK;
    if (!Q || !K || !V || !u_tail || !v_tail || !dO || !dQ || !dK || !dV || !workspace)
        return EOT_ERR_INVALID_ARGUMENT;
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return EOT_ERR_INVALID_ARGUMENT;
    if (workspace_bytes < ws_layout(*p, true).total) return EOT_ERR_WORKSPACE_TOO_SMALL;
    return backward_impl(p, Q, K, V, mask, u_tail, v_tail, dO, dQ, dK, dV, workspace,
                         static_cast<cudaStream_t>(stream));
}

eot_status eot_band_half_step(const eot_problem* p, const void* X, const void* Y, const float* log_marg,
                              const float* in, float* out, void* workspace, size_t workspace_bytes, void* stream) {
    eot_status s = validate(p);
    if (s != EOT_OK) return s;
    if (p->dustbin) return EOT_ERR_UNSUPPORTED;
    if (empty(*p)) return EOT_OK;
    if (!X || !Y || !log_marg || !in || !out || !workspace) return EOT_ERR_INVALID_ARGUMENT;
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return EOT_ERR_INVALID_ARGUMENT;
    if (workspace_bytes < ws_layout(*p, false).total) return EOT_ERR_WORKSPACE_TOO_SMALL;
    return half_step_impl(p, X, Y, log_marg, in, out, workspace, static_cast<cudaStream_t>(stream));
}

eot_status eot_band_half_step_dustbin(const eot_problem* p, const void* X, const void* Y, const float* log_marg,
                                      const float* in, float* out, int32_t own_lo, int32_t own_hi, float* dust_part,
                                      void* workspace, size_t workspace_bytes, void* stream) {
    eot_status s = validate(p);
    if (s != EOT_OK) return s;
    if (!p->dustbin) return EOT_ERR_INVALID_ARGUMENT;
    if (own_lo < 0 || own_hi < own_lo || own_hi > p->dustbin_index) return EOT_ERR_INVALID_ARGUMENT;
    if (empty(*p)) return EOT_OK;
    if (!X || !Y || !log_marg || !in || !out || !dust_part || !workspace) return EOT_ERR_INVALID_ARGUMENT;
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return EOT_ERR_INVALID_ARGUMENT;
    if (workspace_bytes < ws_layout(*p, false).total) return EOT_ERR_WORKSPACE_TOO_SMALL;
    return half_step_impl(p, X, Y, log_marg, in, out, workspace, static_cast<cudaStream_t>(stream), own_lo, own_hi,
                          dust_part);
}

eot_status eot_band_output(const eot_problem* p, const void* Q, const void* K, const void* V, const float* log_marg,
                           const float* u, const float* v, void* O, void* workspace, size_t workspace_bytes,
                           void* stream) {
    eot_status s = validate(p);
    if (s != EOT_OK) return s;
    if (p->dustbin) return EOT_ERR_UNSUPPORTED;
    if (empty(*p)) return EOT_OK;
    if (!Q || !K || !V || !log_marg || !u || !v || !O || !workspace) return EOT_ERR_INVALID_ARGUMENT;
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return EOT_ERR_INVALID_ARGUMENT;
    if (workspace_bytes < ws_layout(*p, false).total) return EOT_ERR_WORKSPACE_TOO_SMALL;
    return output_impl(p, Q, K, V, log_marg, u, v, O, workspace, static_cast<cudaStream_t>(stream));
}

int eot_solve_exp_passes(const eot_problem* p) {
    if (validate(p) != EOT_OK) return -1;
    const Geom g = make_geom(*p);
    if (resolve_impl(*p) == EOT_IMPL_TCGEN05 && g_fwd_schedule.load() >= 2 && iter_schedule_possible(*p) &&
        iter_split(g) > 0)
        return p->T + p->R + 1;   // the first row half-step, then one per iteration
    // every half-step evaluates one exponential per band entry
    return 2 * (p->T + p->R);
}

eot_status eot_set_backward_schedule(int schedule) {
    if (schedule < 0 || schedule > 1) return EOT_ERR_INVALID_ARGUMENT;
    g_bwd_schedule.store(schedule);
    return EOT_OK;
}

eot_status eot_set_forward_schedule(int schedule) {
    if (schedule < 0 || schedule > 3) return EOT_ERR_INVALID_ARGUMENT;
    g_fwd_schedule.store(schedule);
    return EOT_OK;
}

long long eot_kernel_launches(void) { return g_launches.load(); }

void eot_profile_begin(void) {
    g_prof.on = true;
    for (int k = 0; k < kProfKinds; ++k) {
        g_prof.used[k] = 0;
        g_prof.ms[k] = 0.0;
        g_prof.count[k] = 0;
    }
}

eot_status eot_profile_end(void* stream) {
    g_prof.on = false;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return EOT_ERR_CUDA;
    for (int k = 0; k < kProfKinds; ++k) {
        double t = 0.0;
        for (size_t i = 0; i + 1 < g_prof.used[k]; i += 2) {
            float ms = 0.f;
            if (cudaEventElapsedTime(&ms, g_prof.ev[k][i], g_prof.ev[k][i + 1]) != cudaSuccess) return EOT_ERR_CUDA;
            t += ms;
        }
        g_prof.ms[k] = t;
    }
    return EOT_OK;
}

eot_status eot_profile_read(int kind, double* total_ms, long long* launches) {
    if (kind < 0 || kind >= kProfKinds || !total_ms || !launches) return EOT_ERR_INVALID_ARGUMENT;
    *total_ms = g_prof.ms[kind];
    *launches = g_prof.count[kind];
    return EOT_OK;
}

eot_status eot_device_status_bits(void* workspace, void* stream, uint32_t* bits) {
    if (!workspace || !bits) return EOT_ERR_INVALID_ARGUMENT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return EOT_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return EOT_ERR_CUDA;
    *bits = v;
    return EOT_OK;
}

eot_status eot_sq_norms(const void* a, const void* b, size_t n, eot_dtype dtype, double* out, void* stream) {
    if (!out || (n > 0 && (!a || !b)) || (dtype != EOT_FP32 && dtype != EOT_BF16)) return EOT_ERR_INVALID_ARGUMENT;
    int dev = 0, n_sm = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const cudaError_t e = aux(st, [&] { return eot::launch_sq_norms(a, b, n, int(dtype), out, n_sm, st); });
    return e == cudaSuccess ? EOT_OK : EOT_ERR_CUDA;
}

int eot_contraction_offsets(const eot_problem* p) {
    if (validate(p) != EOT_OK) return -1;
    const int h = p->W / 2;
    return h >= 127 ? 2 * ((h - 127) / 128) + 1 : 0;
}

eot_status eot_contraction(const eot_problem* p, const void* Q, const void* K, const uint8_t* mask, float* kappa,
                           void* stream) {
    eot_status s = validate(p);
    if (s != EOT_OK) return s;
    if (empty(*p)) return EOT_OK;
    if (!Q || !K || !kappa) return EOT_ERR_INVALID_ARGUMENT;
    const int n_off = eot_contraction_offsets(p);
    if (n_off == 0) return EOT_OK;
    eot::ContractArgs a{};
    a.Q = Q;
    a.K = K;
    a.mask = mask;
    a.H = p->H;
    a.L = p->L;
    a.d = p->d;
    a.nT = (p->L + 127) / 128;
    a.m = (n_off - 1) / 2;
    a.D = p->dustbin ? p->dustbin_index : -1;
    a.scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf(float(p->d));
    a.kappa = kappa;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const cudaError_t e = aux(st, [&] { return eot::launch_contraction(a, int(p->dtype), p->B * p->H, st); });
    return e == cudaSuccess ? EOT_OK : EOT_ERR_CUDA;
}

eot_status eot_last_device_status(void* workspace, void* stream) {
    uint32_t bits = 0;
    eot_status s = eot_device_status_bits(workspace, stream, &bits);
    if (s != EOT_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), st) != cudaSuccess) return EOT_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return EOT_ERR_CUDA;
    if (bits & kStatusTimeout) return EOT_ERR_TIMEOUT;
    if (bits & kStatusNonFinite) return EOT_ERR_NONFINITE;
    return EOT_OK;
}

}  // extern "C"
