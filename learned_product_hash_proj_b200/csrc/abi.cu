// abi.cu -- the C-ABI: plan validation, workspace layout and the entry
// points that launch the kernels.  Host code only; every step of the mixer
// runs in the kernels of the other files.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>

#include "internal.cuh"

using namespace mono;

namespace {
std::atomic<unsigned long long> g_launches{0};
}

void mono::count_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

namespace {

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

int validate(const mono_config *c) {
    if (c->B < 0 || c->S < 0 || c->W < 1 || c->H < 1 || c->d < 2 || (c->d & 1)) return MONO_ERR_INVALID;
    if (c->Bs < 1 || (c->S % c->Bs) != 0) return MONO_ERR_INVALID;
    if (c->L < 1 || c->R < 0 || c->E < c->R || c->M < 1 || c->C < 1 || c->T < 1 || c->cap < 1) return MONO_ERR_INVALID;
    if (c->d % c->M != 0) return MONO_ERR_INVALID;
    if (!(c->rope_theta > 0.0) || !isfinite(c->rope_theta)) return MONO_ERR_INVALID;
    if (c->dtype != MONO_F32 && c->dtype != MONO_BF16) return MONO_ERR_INVALID;
    long double A = 1;
    for (int m = 0; m < c->M; ++m) A *= c->C;
    if ((long double)c->T > A) return MONO_ERR_INVALID;
    // what this build implements
    if (c->d != 64 && c->d != 128) return MONO_ERR_UNSUPPORTED;
    if (c->M > kMaxM || c->C > kMaxC || c->T > kMaxT || c->E > kMaxE || c->R > kMaxR) return MONO_ERR_UNSUPPORTED;
    if (A > (long double)(1u << 30)) return MONO_ERR_UNSUPPORTED;
    if (c->Bs > 1024) return MONO_ERR_UNSUPPORTED;
    if (c->S / c->Bs > kMaxNb) return MONO_ERR_UNSUPPORTED;
    if (c->W % 64 != 0) return MONO_ERR_UNSUPPORTED;
    if ((long long)c->B * c->H * c->S * c->d > (1ll << 40)) return MONO_ERR_UNSUPPORTED;
    if ((c->flags & MONO_FLAG_REDIRECT) && A > (long double)kRedirectMaxA) return MONO_ERR_UNSUPPORTED;
    if (c->flags & ~(MONO_FLAG_SIMPLE_KERNELS | MONO_FLAG_REDIRECT)) return MONO_ERR_INVALID;
    return MONO_OK;
}

void layout(Plan *p) {
    const mono_config &c = p->cfg;
    const size_t B = c.B, H = c.H, S = c.S, d = c.d, nb = p->nb, R = c.R, es = p->es;
    size_t bytes[kRegN] = {};
    bytes[kRegKbar] = B * H * nb * d * 4;
    bytes[kRegAddr] = B * H * nb * 4;
    bytes[kRegPostIds] = B * H * nb * 4;
    bytes[kRegPostAddr] = B * H * nb * 4;
    bytes[kRegPostRank] = B * H * nb * 4;
    bytes[kRegOverflow] = B * H * 4;
    bytes[kRegQ] = B * H * S * d * es;
    bytes[kRegK] = B * H * S * d * es;
    bytes[kRegV] = B * H * S * d * es;
    bytes[kRegSel] = B * H * S * R * 4;
    bytes[kRegO] = B * S * H * d * es;
    bytes[kRegCounters] = kCntN * 8;
    bytes[kRegWalkLog] = kWalkLogCap * 4;
    const size_t nhi = (S + kRopeLo - 1) / kRopeLo;
    bytes[kRegRope] = (nhi + kRopeLo) * (d / 2) * 8;
    if (p->fast && R > 0) {
        bytes[kRegPairCount] = B * H * nb * 4;
        bytes[kRegPairStart] = B * H * nb * 4;
        bytes[kRegPairFill] = B * H * nb * 4;
        bytes[kRegPairs] = B * H * S * R * 4;
        bytes[kRegPartO] = B * H * S * R * d * 2;
        bytes[kRegPartML] = B * H * S * R * 8;
        bytes[kRegWork] = B * H * (size_t)p->max_work * 16;
        bytes[kRegNWork] = B * H * 4;
    }
    size_t off = 0;
    for (int r = 0; r < kRegN; ++r) {
        p->off[r] = off;
        p->bytes[r] = bytes[r];
        off = align_up(off + bytes[r], 256);
    }
    p->ws_bytes = off;
}

bool empty(const Plan *p) { return p->cfg.B == 0 || p->cfg.S == 0; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? MONO_OK : MONO_ERR_CUDA; }

int check_common(const mono_plan_t *plan, const void *ws) {
    if (!plan) return MONO_ERR_NULL;
    if (!ws) return MONO_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return MONO_ERR_ALIGN;
    return MONO_OK;
}

int check_ptrs(std::initializer_list<const void *> ptrs) {
    for (const void *q : ptrs) {
        if (!q) return MONO_ERR_NULL;
        if (!aligned(q, 16)) return MONO_ERR_ALIGN;
    }
    return MONO_OK;
}

}  // namespace

extern "C" {

int mono_version(void) { return MONO_VERSION; }

unsigned long long mono_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

const char *mono_strerror(int s) {
    switch (s) {
        case MONO_OK: return "ok";
        case MONO_ERR_INVALID: return "parameters violate the method's definition";
        case MONO_ERR_UNSUPPORTED: return "parameters outside what this build implements";
        case MONO_ERR_NULL: return "a required pointer is NULL";
        case MONO_ERR_WORKSPACE: return "workspace missing";
        case MONO_ERR_CUDA: return "a CUDA call or kernel launch failed";
        case MONO_ERR_DEVICE: return "a kernel recorded a device error";
        case MONO_ERR_ALIGN: return "a pointer is not suitably aligned";
        case MONO_ERR_SCRATCH: return "problem too large for the fixed scratch array of mono_route_static";
        default: return "unknown status";
    }
}

int mono_plan(const mono_config *cfg, mono_plan_t **plan, size_t *workspace_bytes) {
    if (!cfg || !plan) return MONO_ERR_NULL;
    *plan = nullptr;
    int v = validate(cfg);
    if (v != MONO_OK) return v;
    mono_plan_s *ps = (mono_plan_s *)calloc(1, sizeof(mono_plan_s));
    if (!ps) return MONO_ERR_INVALID;
    Plan &p = ps->p;
    p.cfg = *cfg;
    p.nb = cfg->S / cfg->Bs;
    p.A = 1;
    for (int m = 0; m < cfg->M; ++m) p.A *= cfg->C;
    p.es = cfg->dtype == MONO_BF16 ? 2 : 4;
    p.fast = attend_tc_supported(*cfg) && !(cfg->flags & MONO_FLAG_SIMPLE_KERNELS);
    p.gemm_tc = gemm_tc_supported(*cfg) && !(cfg->flags & MONO_FLAG_SIMPLE_KERNELS);
    {
        // remote work items per (b, h): one per bucket at most, plus one per 128 pairs
        const long long mw = (long long)p.nb + ((long long)cfg->S * cfg->R + 127) / 128;
        if (p.fast && cfg->R > 0 && mw > (1ll << 31) - 1) { free(ps); return MONO_ERR_UNSUPPORTED; }
        p.max_work = (int)(mw < (1ll << 31) - 1 ? mw : 0);
    }
    layout(&p);
    *plan = ps;
    if (workspace_bytes) *workspace_bytes = p.ws_bytes;
    return MONO_OK;
}

void mono_plan_destroy(mono_plan_t *plan) { free(plan); }

int mono_workspace_region(const mono_plan_t *plan, int region, size_t *offset, size_t *bytes) {
    if (!plan || !offset || !bytes) return MONO_ERR_NULL;
    if (region < 0 || region >= MONO_WS_NREGIONS) return MONO_ERR_INVALID;
    *offset = plan->p.off[region];
    *bytes = plan->p.bytes[region];
    return MONO_OK;
}

int mono_project(const mono_plan_t *plan, const void *x, const void *Wq, const void *Wk, const void *Wv, void *Q,
                 void *K, void *V, void *workspace, void *stream) {
    int st = check_common(plan, workspace);
    if (st) return st;
    const Plan &p = plan->p;
    if (empty(&p)) return MONO_OK;
    if ((st = check_ptrs({x, Wq, Wk, Wv, Q, K, V}))) return st;
    cudaStream_t s = (cudaStream_t)stream;
    if ((st = cuda_status(launch_rope_tables(p, workspace, s)))) return st;
    if (p.gemm_tc) return cuda_status(launch_project_tc(p, x, Wq, Wk, Wv, Q, K, V, workspace, s));
    return cuda_status(launch_project_simt(p, x, Wq, Wk, Wv, Q, K, V, workspace, s));
}

int mono_route_summaries(const mono_plan_t *plan, const void *K, const float *codebooks, void *workspace,
                         void *stream) {
    int st = check_common(plan, workspace);
    if (st) return st;
    const Plan &p = plan->p;
    if (empty(&p)) return MONO_OK;
    if ((st = check_ptrs({K, codebooks}))) return st;
    return cuda_status(launch_summaries(p, K, codebooks, workspace, (cudaStream_t)stream));
}

int mono_route_lists(const mono_plan_t *plan, void *workspace, void *stream) {
    int st = check_common(plan, workspace);
    if (st) return st;
    const Plan &p = plan->p;
    if (empty(&p)) return MONO_OK;
    return cuda_status(launch_lists(p, workspace, (cudaStream_t)stream));
}

int mono_route_queries(const mono_plan_t *plan, const void *Q, const float *codebooks, const int32_t *forced,
                       int32_t *sel, void *workspace, void *stream) {
    int st = check_common(plan, workspace);
    if (st) return st;
    const Plan &p = plan->p;
    if (empty(&p)) return MONO_OK;
    if ((st = check_ptrs({Q, codebooks}))) return st;
    if (p.cfg.R > 0 && (st = check_ptrs({sel}))) return st;
    if (forced && !aligned(forced, 4)) return MONO_ERR_ALIGN;
    return cuda_status(launch_queries(p, Q, codebooks, forced, sel, workspace, (cudaStream_t)stream));
}

int mono_route(const mono_plan_t *plan, const void *Q, const void *K, const float *codebooks, const int32_t *forced,
               int32_t *sel, void *workspace, void *stream) {
    int st = check_common(plan, workspace);
    if (st) return st;
    const Plan &p = plan->p;
    if (empty(&p)) return MONO_OK;
    if ((st = check_ptrs({Q, K, codebooks}))) return st;
    if (p.cfg.R > 0 && (st = check_ptrs({sel}))) return st;
    if (forced && !aligned(forced, 4)) return MONO_ERR_ALIGN;
    if ((st = mono_route_summaries(plan, K, codebooks, workspace, stream))) return st;
    if ((st = mono_route_lists(plan, workspace, stream))) return st;
    // the lists launch cleared the statistics: the probe follows it directly (programmatic launch)
    return cuda_status(launch_queries(p, Q, codebooks, forced, sel, workspace, (cudaStream_t)stream, false));
}

int mono_attend(const mono_plan_t *plan, const void *Q, const void *K, const void *V, const int32_t *sel, void *O,
                void *workspace, void *stream) {
    int st = check_common(plan, workspace);
    if (st) return st;
    const Plan &p = plan->p;
    if (empty(&p)) return MONO_OK;
    if ((st = check_ptrs({Q, K, V, O}))) return st;
    if (p.cfg.R > 0 && (st = check_ptrs({sel}))) return st;
    cudaStream_t s = (cudaStream_t)stream;
    if (p.fast) return cuda_status(launch_attend_tc(p, Q, K, V, sel, O, workspace, s));
    return cuda_status(launch_attend_simt(p, Q, K, V, sel, O, workspace, s));
}

static int attend_part(const mono_plan_t *plan, const void *Q, const void *K, const void *V, const int32_t *sel,
                       void *O, void *workspace, void *stream, int parts) {
    int st = check_common(plan, workspace);
    if (st) return st;
    const Plan &p = plan->p;
    if (empty(&p)) return MONO_OK;
    cudaStream_t s = (cudaStream_t)stream;
    if (!p.fast) {  // one query-major kernel does the whole attention: it runs as the local stage
        if (!(parts & kAttendLocal)) return MONO_OK;
        if ((st = check_ptrs({Q, K, V, O}))) return st;
        if (p.cfg.R > 0 && (st = check_ptrs({sel}))) return st;
        return cuda_status(launch_attend_simt(p, Q, K, V, sel, O, workspace, s));
    }
    if ((parts & (kAttendRemote | kAttendLocal)) && (st = check_ptrs({Q, K, V}))) return st;
    if ((parts & kAttendLocal) && (st = check_ptrs({O}))) return st;
    if (p.cfg.R > 0 && (parts & (kAttendPairs | kAttendLocal)) && (st = check_ptrs({sel}))) return st;
    return cuda_status(launch_attend_tc(p, Q, K, V, sel, O, workspace, s, parts));
}

int mono_attend_pairs(const mono_plan_t *plan, const int32_t *sel, void *workspace, void *stream) {
    return attend_part(plan, nullptr, nullptr, nullptr, sel, nullptr, workspace, stream, kAttendPairs);
}

int mono_attend_remote(const mono_plan_t *plan, const void *Q, const void *K, const void *V, void *workspace,
                       void *stream) {
    return attend_part(plan, Q, K, V, nullptr, nullptr, workspace, stream, kAttendRemote);
}

int mono_attend_local(const mono_plan_t *plan, const void *Q, const void *K, const void *V, const int32_t *sel,
                      void *O, void *workspace, void *stream) {
    return attend_part(plan, Q, K, V, sel, O, workspace, stream, kAttendLocal);
}

int mono_out_project(const mono_plan_t *plan, const void *O, const void *Wo, void *delta, void *workspace,
                     void *stream) {
    int st = check_common(plan, workspace);
    if (st) return st;
    const Plan &p = plan->p;
    if (empty(&p)) return MONO_OK;
    if ((st = check_ptrs({O, Wo, delta}))) return st;
    if (p.gemm_tc) return cuda_status(launch_out_project_tc(p, O, Wo, delta, workspace, (cudaStream_t)stream));
    return cuda_status(launch_out_project_simt(p, O, Wo, delta, (cudaStream_t)stream));
}

int mono_out_project_scatter(const mono_plan_t *plan, const void *O, const void *Wo, float *const *stage,
                             int nranks, int rank, void *workspace, void *stream) {
    int st = check_common(plan, workspace);
    if (st) return st;
    const Plan &p = plan->p;
    if (!stage) return MONO_ERR_NULL;
    if (nranks < 1 || nranks > 8 || rank < 0 || rank >= nranks) return MONO_ERR_INVALID;
    if (((long long)p.cfg.B * p.cfg.S) % nranks) return MONO_ERR_INVALID;
    if (!p.gemm_tc) return MONO_ERR_UNSUPPORTED;
    if (empty(&p)) return MONO_OK;
    if ((st = check_ptrs({O, Wo}))) return st;
    for (int r = 0; r < nranks; ++r)
        if ((st = check_ptrs({stage[r]}))) return st;
    return cuda_status(launch_out_project_stage(p, O, Wo, stage, nranks, rank, workspace, (cudaStream_t)stream));
}

int mono_stage_reduce(const mono_plan_t *plan, const float *stage, int nranks, void *delta_chunk, void *stream) {
    if (!plan) return MONO_ERR_NULL;
    const Plan &p = plan->p;
    if (nranks < 1 || nranks > 8) return MONO_ERR_INVALID;
    if (((long long)p.cfg.B * p.cfg.S) % nranks) return MONO_ERR_INVALID;
    if (!p.gemm_tc) return MONO_ERR_UNSUPPORTED;
    if (empty(&p)) return MONO_OK;
    int st;
    if ((st = check_ptrs({stage, delta_chunk}))) return st;
    return cuda_status(launch_stage_reduce(p, stage, nranks, delta_chunk, (cudaStream_t)stream));
}

int mono_forward(const mono_plan_t *plan, const void *x, const void *Wq, const void *Wk, const void *Wv,
                 const void *Wo, const float *codebooks, const int32_t *forced, void *delta, void *workspace,
                 void *stream) {
    int st = check_common(plan, workspace);
    if (st) return st;
    const Plan &p = plan->p;
    if (empty(&p)) return MONO_OK;
    if ((st = check_ptrs({x, Wq, Wk, Wv, Wo, codebooks, delta}))) return st;
    void *Q = ws_ptr(p, workspace, kRegQ), *K = ws_ptr(p, workspace, kRegK), *V = ws_ptr(p, workspace, kRegV);
    int32_t *sel = (int32_t *)ws_ptr(p, workspace, kRegSel);
    void *O = ws_ptr(p, workspace, kRegO);
    if ((st = mono_project(plan, x, Wq, Wk, Wv, Q, K, V, workspace, stream))) return st;
    if ((st = mono_route(plan, Q, K, codebooks, forced, sel, workspace, stream))) return st;
    if ((st = mono_attend(plan, Q, K, V, sel, O, workspace, stream))) return st;
    return mono_out_project(plan, O, Wo, delta, workspace, stream);
}

int mono_stats(const mono_plan_t *plan, const void *workspace, void *stream, mono_stats_t *out) {
    if (!plan || !out) return MONO_ERR_NULL;
    memset(out, 0, sizeof(*out));
    if (empty(&plan->p)) return MONO_OK;
    // NULL workspace: the tables mono_route_static left in its fixed array
    Plan rp;
    const bool from_static = workspace == nullptr;
    if (from_static) {
        void *base = nullptr;
        const int st = route_static_tables(plan->p, &base, &rp);
        if (st != MONO_OK) return st;
        workspace = base;
    }
    const Plan &p = from_static ? rp : plan->p;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MONO_ERR_CUDA;
    unsigned long long cnt[kCntN];
    const size_t nbh = (size_t)p.cfg.B * p.cfg.H;
    int32_t *ov = (int32_t *)malloc(nbh * sizeof(int32_t));
    if (!ov) return MONO_ERR_CUDA;
    cudaError_t e1 = cudaMemcpy(cnt, (const char *)workspace + p.off[kRegCounters], sizeof(cnt), cudaMemcpyDeviceToHost);
    cudaError_t e2 = cudaMemcpy(ov, (const char *)workspace + p.off[kRegOverflow], nbh * 4, cudaMemcpyDeviceToHost);
    if (e1 != cudaSuccess || e2 != cudaSuccess) { free(ov); return MONO_ERR_CUDA; }
    for (size_t i = 0; i < nbh; ++i) {
        out->overflow_total += ov[i];
        if (ov[i] > out->overflow_max_bh) out->overflow_max_bh = ov[i];
    }
    free(ov);
    out->queries_lt_R = (int64_t)cnt[kCntQueriesLtR];
    out->remote_selected = (int64_t)cnt[kCntRemoteSel];
    out->forced_ignored = (int64_t)cnt[kCntForcedIgnored];
    out->probe_walks = (int64_t)cnt[kCntWalks];
    out->device_error = (int32_t)cnt[kCntErr];
    out->mean_remote = (double)out->remote_selected / ((double)p.cfg.B * p.cfg.H * p.cfg.S);
    return out->device_error ? MONO_ERR_DEVICE : MONO_OK;
}

}  // extern "C"
