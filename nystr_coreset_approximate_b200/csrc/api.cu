// api.cu -- extern "C" entry points of libwildcat (declared in include/wildcat.h).
//
// Host-side argument checks, workspace carving and stage sequencing.  No
// arithmetic of the method happens here; every stage runs in the kernels of
// select.cu, weights.cu and attend.cu.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>

#include "../../include/wildcat.h"
#include "internal.h"

using wildcat::Carve;
using wildcat::Status;

namespace {

thread_local char g_err[512] = "";

wildcat_status record(const Status& s) {
    if (s.code == 0) {
        g_err[0] = '\0';
        return WILDCAT_OK;
    }
    if (s.code == WILDCAT_ERR_CUDA)
        snprintf(g_err, sizeof(g_err), "%s: %s", s.what, cudaGetErrorString(s.cuda_err));
    else
        snprintf(g_err, sizeof(g_err), "%s", s.what);
    return (wildcat_status)s.code;
}

wildcat_status bad(int code, const char* fmt, const char* what) {
    snprintf(g_err, sizeof(g_err), fmt, what);
    return (wildcat_status)code;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t elem_bytes(int dtype) { return dtype == WILDCAT_BF16 ? 2 : 4; }

wildcat_status check_common(int dtype, int64_t BH, int64_t n, int d, int r, const char* who) {
    if (dtype != WILDCAT_F32 && dtype != WILDCAT_BF16) return bad(1, "%s: dtype must be WILDCAT_F32 or WILDCAT_BF16", who);
    if (BH < 0) return bad(1, "%s: BH must be >= 0", who);
    if (n < 1) return bad(1, "%s: n must be >= 1", who);
    if (r < 1 || (int64_t)r > n) return bad(1, "%s: r must satisfy 1 <= r <= n", who);
    if (d != 32 && d != 64 && d != 128) return bad(2, "%s: head dim must be 32, 64 or 128", who);
    if (r > 8192) return bad(2, "%s: r above 8192 is not supported", who);
    const double cells = (double)BH * (double)n * (double)(d > r ? d : r);
    if (cells > 4.0e18) return bad(1, "%s: tensor sizes overflow 64-bit offsets", who);
    if (BH > 65535) return bad(2, "%s: BH above 65535 is not supported", who);
    return WILDCAT_OK;
}

wildcat_status check_scalars(float beta, float eps, const char* who) {
    if (!std::isfinite(beta) || !(beta > 0.f)) return bad(1, "%s: beta must be finite and > 0", who);
    if (!std::isfinite(eps) || eps < 0.f) return bad(1, "%s: eps must be finite and >= 0", who);
    return WILDCAT_OK;
}

wildcat_status select_impl(const void* K, int dtype, int64_t BH, int64_t n, int d, float beta, int r, uint64_t seed,
                           int64_t inst0, float eps, const int32_t* S_fixed, int32_t* S, float* F, int32_t* rank,
                           void* K_S, void* stream, const char* who, void* ws = nullptr, size_t ws_bytes = 0) {
    wildcat_status st = check_common(dtype, BH, n, d, r, who);
    if (st != WILDCAT_OK) return st;
    if ((st = check_scalars(beta, eps, who)) != WILDCAT_OK) return st;
    if (inst0 < 0 || inst0 + BH > 4294967296LL) return bad(1, "%s: inst0 must satisfy 0 <= inst0, inst0 + BH <= 2^32", who);
    if (BH == 0) return record(Status::ok());
    if (!K || !F || !rank) return bad(1, "%s: K, F and rank must be non-null", who);
    if (!S_fixed && !S) return bad(1, "%s: S must be non-null", who);
    if (!aligned16(K) || !aligned16(F) || (K_S && !aligned16(K_S)))
        return bad(1, "%s: K, F and K_S must be 16-byte aligned", who);
    if (ws && (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return bad(4, "%s: workspace must be 256-byte aligned", who);
    wildcat::SelectRequest q{K, dtype, BH, n, d, beta, r, seed, inst0, eps, S_fixed, S, F, rank, K_S};
    q.ws = ws;
    q.ws_bytes = ws_bytes;
    return record(wildcat::launch_select(q, static_cast<cudaStream_t>(stream)));
}

struct ForwardLayout {
    float* F;
    int32_t* S;
    int32_t* rank;
    void* K_S;
    float* V_S;
    float* w;
    float* vmin;
    float* vmax;
    void* wws;
    size_t wws_bytes;
    void* aws;
    size_t aws_bytes;
    void* sws;  // select workspace (global-sync mode)
    size_t sws_bytes;
    void* rws;  // value-range partials (their own region: the range runs beside the select)
    size_t rws_bytes;
};

ForwardLayout carve_forward(Carve& cv, int64_t BH, int64_t m, int64_t n, int d, int r, int dtype) {
    ForwardLayout L{};
    L.F = static_cast<float*>(cv.take(sizeof(float) * BH * (int64_t)r * n));
    L.S = static_cast<int32_t*>(cv.take(sizeof(int32_t) * BH * r));
    L.rank = static_cast<int32_t*>(cv.take(sizeof(int32_t) * BH));
    L.K_S = cv.take(elem_bytes(dtype) * BH * (int64_t)r * d);
    L.V_S = static_cast<float*>(cv.take(sizeof(float) * BH * (int64_t)r * d));
    L.w = static_cast<float*>(cv.take(sizeof(float) * BH * r));
    L.vmin = static_cast<float*>(cv.take(sizeof(float) * BH * d));
    L.vmax = static_cast<float*>(cv.take(sizeof(float) * BH * d));
    L.wws_bytes = wildcat::weights_workspace_bytes(BH, n, d, r);
    L.wws = cv.take(L.wws_bytes);
    L.aws_bytes = wildcat::attend_workspace_bytes(BH, m, d, r);
    L.aws = cv.take(L.aws_bytes);
    L.sws_bytes = wildcat::select_workspace_bytes(BH, n);
    L.sws = cv.take(L.sws_bytes);
    L.rws_bytes = wildcat::value_range_workspace_bytes(BH, n, d);
    L.rws = cv.take(L.rws_bytes);
    return L;
}

// One auxiliary stream and two events per device, created on first use: a
// forward runs the value range of V there, beside its select (only the
// attend needs v_min / v_max).  A forward holds the device's mutex from the
// fork to the join, so calls from several threads do not mix the events.
struct AuxPipe {
    std::mutex mu;
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};

AuxPipe* aux_pipe() {
    static std::mutex pool_mu;
    static std::map<int, AuxPipe*> pool;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(pool_mu);
    auto it = pool.find(dev);
    if (it != pool.end()) return it->second;
    AuxPipe* ap = new AuxPipe();
    bool ok = cudaStreamCreateWithFlags(&ap->s, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&ap->fork, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&ap->join, cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
        cudaGetLastError();
        delete ap;  // the handles that were created are left to the context's teardown
        return nullptr;
    }
    pool[dev] = ap;
    return ap;
}

// Starts the value range of V [BH, n, d] on the device's auxiliary stream
// after the work queued on `st` (and after `wait_v` when given), so that it
// runs beside the select.  Returns with `lock` holding the device's mutex and
// *forked set; join_value_range makes `st` wait for the range.  Without an
// auxiliary stream (*forked false) the caller forms the range on `st`.
Status fork_value_range(const void* V, int dtype, int64_t BH, int64_t n, int d, float* vmin, float* vmax, void* ws,
                        size_t ws_bytes, cudaStream_t st, cudaEvent_t wait_v, std::unique_lock<std::mutex>& lock,
                        AuxPipe** ap_out, bool* forked) {
    *forked = false;
    AuxPipe* ap = aux_pipe();
    *ap_out = ap;
    if (!ap) return Status::ok();
    lock = std::unique_lock<std::mutex>(ap->mu);
    cudaError_t e;
    if ((e = cudaEventRecord(ap->fork, st))) return Status::cuda(e, "forward: fork");
    if ((e = cudaStreamWaitEvent(ap->s, ap->fork, 0))) return Status::cuda(e, "forward: fork");
    if (wait_v && (e = cudaStreamWaitEvent(ap->s, wait_v, 0))) return Status::cuda(e, "forward: wait for V");
    const Status z = wildcat::launch_value_range(V, dtype, BH, n, d, vmin, vmax, ws, ws_bytes, ap->s);
    if (z.code) return z;
    if ((e = cudaEventRecord(ap->join, ap->s))) return Status::cuda(e, "forward: join");
    *forked = true;
    return Status::ok();
}

Status join_value_range(AuxPipe* ap, cudaStream_t st, std::unique_lock<std::mutex>& lock) {
    const cudaError_t e = cudaStreamWaitEvent(st, ap->join, 0);
    lock.unlock();
    return e ? Status::cuda(e, "forward: join") : Status::ok();
}

// Stage markers (wildcat_set_stage_events): caller-owned events recorded on
// a forward's stream right after its select and right after its weights.
thread_local cudaEvent_t g_ev_after_select = nullptr;
thread_local cudaEvent_t g_ev_after_weights = nullptr;
static Status mark_stage(cudaEvent_t ev, cudaStream_t st, const char* what) {
    if (!ev) return Status::ok();
    const cudaError_t e = cudaEventRecord(ev, st);
    return e == cudaSuccess ? Status::ok() : Status::cuda(e, what);
}

// wait_v / wait_q (optional): events the weights / attend stage waits for
// (the host-buffer forward copies V and Q while the select runs).
wildcat_status forward_impl(const void* Q, const void* K, const void* V, int dtype, int64_t BH, int64_t m, int64_t n,
                            int d, float beta, int r, uint64_t seed, int64_t inst0, float eps, float* O,
                            int32_t* S_out, int32_t* rank_out, const ForwardLayout& L, cudaStream_t st,
                            cudaEvent_t wait_v = nullptr, cudaEvent_t wait_q = nullptr) {
    Status s;
    cudaError_t ew;
    std::unique_lock<std::mutex> aux_lock;
    AuxPipe* ap = nullptr;
    bool forked = false;
    if ((s = fork_value_range(V, dtype, BH, n, d, L.vmin, L.vmax, L.rws, L.rws_bytes, st, wait_v, aux_lock, &ap,
                              &forked)).code)
        return record(s);
    wildcat::SelectRequest sq{K, dtype, BH, n, d, beta, r, seed, inst0, eps, nullptr, L.S, L.F, L.rank, L.K_S};
    sq.ws = L.sws;
    sq.ws_bytes = L.sws_bytes;
    if ((s = wildcat::launch_select(sq, st)).code) return record(s);
    if ((s = mark_stage(g_ev_after_select, st, "forward: stage event")).code) return record(s);
    if (wait_v && (ew = cudaStreamWaitEvent(st, wait_v, 0))) return record(Status::cuda(ew, "forward: wait for V"));
    wildcat::WeightsRequest wq{L.F, L.S, L.rank, V, dtype, BH, n, d, r, L.V_S, L.w, L.vmin, L.vmax, L.wws,
                               L.wws_bytes};
    wq.skip_range = forked;
    if ((s = wildcat::launch_weights(wq, st)).code) return record(s);
    if ((s = mark_stage(g_ev_after_weights, st, "forward: stage event")).code) return record(s);
    if (forked && (s = join_value_range(ap, st, aux_lock)).code) return record(s);
    if (wait_q && (ew = cudaStreamWaitEvent(st, wait_q, 0))) return record(Status::cuda(ew, "forward: wait for Q"));
    if (m > 0) {
        wildcat::AttendRequest aq{Q,   L.K_S,  dtype, BH, m, d, r, L.rank, beta, L.V_S, L.w,
                                  L.vmin, L.vmax, O,   L.aws, L.aws_bytes};
        if ((s = wildcat::launch_attend(aq, st)).code) return record(s);
    }
    cudaError_t e;
    if (S_out && (e = cudaMemcpyAsync(S_out, L.S, sizeof(int32_t) * BH * r, cudaMemcpyDeviceToDevice, st)))
        return record(Status::cuda(e, "forward: copy S"));
    if (rank_out && (e = cudaMemcpyAsync(rank_out, L.rank, sizeof(int32_t) * BH, cudaMemcpyDeviceToDevice, st)))
        return record(Status::cuda(e, "forward: copy rank"));
    return record(Status::ok());
}

struct BinnedLayout {
    float* F;
    int32_t* S;
    int32_t* rank_b;
    void* K_S;
    float* V_S;
    float* w;
    float* vmin_b;
    float* vmax_b;
    float* vmin;
    float* vmax;
    int32_t* rank_att;
    void* wws;
    size_t wws_bytes;
    void* aws;
    size_t aws_bytes;
    float* kbar;   // recentring only
    void* mws;
    void* sws;     // select workspace (global-sync mode)
    size_t sws_bytes;
    void* rws;     // value-range partials of the bins
    size_t rws_bytes;
};

BinnedLayout carve_binned(Carve& cv, int64_t BH, int64_t m, int64_t n, int d, int r, int nbins, int dtype,
                          bool recenter) {
    const int64_t nb = n / nbins;
    const int rb = r / nbins;
    const int64_t BB = BH * nbins;
    BinnedLayout L{};
    L.F = static_cast<float*>(cv.take(sizeof(float) * BB * (int64_t)rb * nb));
    L.S = static_cast<int32_t*>(cv.take(sizeof(int32_t) * BH * r));
    L.rank_b = static_cast<int32_t*>(cv.take(sizeof(int32_t) * BB));
    L.K_S = cv.take(elem_bytes(dtype) * BH * (int64_t)r * d);
    L.V_S = static_cast<float*>(cv.take(sizeof(float) * BH * (int64_t)r * d));
    L.w = static_cast<float*>(cv.take(sizeof(float) * BH * r));
    L.vmin_b = static_cast<float*>(cv.take(sizeof(float) * BB * d));
    L.vmax_b = static_cast<float*>(cv.take(sizeof(float) * BB * d));
    L.vmin = static_cast<float*>(cv.take(sizeof(float) * BH * d));
    L.vmax = static_cast<float*>(cv.take(sizeof(float) * BH * d));
    L.rank_att = static_cast<int32_t*>(cv.take(sizeof(int32_t) * BH));
    L.wws_bytes = wildcat::weights_workspace_bytes(BB, nb, d, rb);
    L.wws = cv.take(L.wws_bytes);
    L.aws_bytes = wildcat::attend_workspace_bytes(BH, m, d, r);
    L.aws = cv.take(L.aws_bytes);
    L.kbar = recenter ? static_cast<float*>(cv.take(sizeof(float) * BH * d)) : nullptr;
    L.mws = recenter ? cv.take(wildcat::key_mean_workspace_bytes(BH, n, d)) : nullptr;
    L.sws_bytes = wildcat::select_workspace_bytes(BB, nb);
    L.sws = cv.take(L.sws_bytes);
    L.rws_bytes = wildcat::value_range_workspace_bytes(BB, nb, d);
    L.rws = cv.take(L.rws_bytes);
    return L;
}

wildcat_status check_bins(int64_t BH, int64_t n, int r, int nbins, const char* who) {
    if (nbins < 1) return bad(1, "%s: nbins must be >= 1", who);
    if (n % nbins || r % nbins) return bad(1, "%s: n and r must be multiples of nbins", who);
    if (BH * nbins > 65535) return bad(2, "%s: BH * nbins above 65535 is not supported", who);
    return WILDCAT_OK;
}

}  // namespace

// One copy stream and four events per device for the host-buffer forward,
// created on first use; a call holds the device's mutex while it runs.
struct HostPipe {
    std::mutex mu;
    cudaStream_t cs = nullptr;
    cudaEvent_t ready = nullptr, k_in = nullptr, v_in = nullptr, q_in = nullptr;
};

HostPipe* host_pipe(int dev) {
    static std::mutex pool_mu;
    static std::map<int, HostPipe*> pool;
    std::lock_guard<std::mutex> lock(pool_mu);
    auto it = pool.find(dev);
    if (it != pool.end()) return it->second;
    HostPipe* hp = new HostPipe();
    bool ok = cudaStreamCreateWithFlags(&hp->cs, cudaStreamNonBlocking) == cudaSuccess;
    for (cudaEvent_t* ev : {&hp->ready, &hp->k_in, &hp->v_in, &hp->q_in})
        ok = ok && cudaEventCreateWithFlags(ev, cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
        cudaGetLastError();
        delete hp;  // the handles that were created are left to the context's teardown
        return nullptr;
    }
    pool[dev] = hp;
    return hp;
}

// Copies K, then V, then Q (host -> device) on the device's copy stream,
// after the work already queued on `s`; `s` waits for K.  The caller holds
// hp->mu and makes its weights and attend stages wait for hp->v_in / hp->q_in.
Status stage_host_inputs(HostPipe* hp, cudaStream_t s, void* Kd, void* Vd, void* Qd, const void* K_host,
                         const void* V_host, const void* Q_host, size_t kv_bytes, size_t q_bytes) {
    cudaError_t e;
    if ((e = cudaEventRecord(hp->ready, s))) return Status::cuda(e, "forward_host: record");
    if ((e = cudaStreamWaitEvent(hp->cs, hp->ready, 0))) return Status::cuda(e, "forward_host: wait");
    if ((e = cudaMemcpyAsync(Kd, K_host, kv_bytes, cudaMemcpyHostToDevice, hp->cs)))
        return Status::cuda(e, "forward_host: copy K");
    if ((e = cudaEventRecord(hp->k_in, hp->cs))) return Status::cuda(e, "forward_host: record");
    if ((e = cudaMemcpyAsync(Vd, V_host, kv_bytes, cudaMemcpyHostToDevice, hp->cs)))
        return Status::cuda(e, "forward_host: copy V");
    if ((e = cudaEventRecord(hp->v_in, hp->cs))) return Status::cuda(e, "forward_host: record");
    if (q_bytes && (e = cudaMemcpyAsync(Qd, Q_host, q_bytes, cudaMemcpyHostToDevice, hp->cs)))
        return Status::cuda(e, "forward_host: copy Q");
    if ((e = cudaEventRecord(hp->q_in, hp->cs))) return Status::cuda(e, "forward_host: record");
    if ((e = cudaStreamWaitEvent(s, hp->k_in, 0))) return Status::cuda(e, "forward_host: wait for K");
    return Status::ok();
}

namespace wildcat {
int read_device_status(bool clear) {
    const int parts[3] = {read_attend_status(clear), read_weights_status(clear), read_select_gs_status(clear)};
    for (const int v : parts)
        if (v < 0) return -1;
    for (const int v : parts)
        if (v) return v;
    return 0;
}
}  // namespace wildcat

extern "C" {

int wildcat_version(void) { return 100; }

const char* wildcat_last_error(void) { return g_err; }

const char* wildcat_status_string(int status) {
    switch (status) {
        case WILDCAT_OK: return "WILDCAT_OK";
        case WILDCAT_ERR_INVALID_ARG: return "WILDCAT_ERR_INVALID_ARG";
        case WILDCAT_ERR_UNSUPPORTED: return "WILDCAT_ERR_UNSUPPORTED";
        case WILDCAT_ERR_CUDA: return "WILDCAT_ERR_CUDA";
        case WILDCAT_ERR_WORKSPACE: return "WILDCAT_ERR_WORKSPACE";
        case WILDCAT_ERR_TIMEOUT: return "WILDCAT_ERR_TIMEOUT";
    }
    return "WILDCAT_UNKNOWN_STATUS";
}

wildcat_status wildcat_select(const void* K, int dtype, int64_t BH, int64_t n, int d, float beta, int r, uint64_t seed,
                              int64_t inst0, float eps, int32_t* S, float* F, int32_t* rank, void* K_S,
                              void* stream) {
    return select_impl(K, dtype, BH, n, d, beta, r, seed, inst0, eps, nullptr, S, F, rank, K_S, stream,
                       "wildcat_select");
}

size_t wildcat_select_workspace_size(int64_t BH, int64_t n) {
    if (BH < 0 || n < 1) return 0;
    return wildcat::select_workspace_bytes(BH, n);
}

wildcat_status wildcat_select_ws(const void* K, int dtype, int64_t BH, int64_t n, int d, float beta, int r,
                                 uint64_t seed, int64_t inst0, float eps, int32_t* S, float* F, int32_t* rank,
                                 void* K_S, void* workspace, size_t ws_bytes, void* stream) {
    return select_impl(K, dtype, BH, n, d, beta, r, seed, inst0, eps, nullptr, S, F, rank, K_S, stream,
                       "wildcat_select_ws", workspace, ws_bytes);
}

wildcat_status wildcat_select_fixed(const void* K, int dtype, int64_t BH, int64_t n, int d, float beta, int r,
                                    float eps, const int32_t* S_fixed, int32_t* S, float* F, int32_t* rank,
                                    void* K_S, void* stream) {
    if (!S_fixed && BH > 0) return bad(1, "%s: S_fixed must be non-null", "wildcat_select_fixed");
    return select_impl(K, dtype, BH, n, d, beta, r, 0, 0, eps, S_fixed, S, F, rank, K_S, stream,
                       "wildcat_select_fixed");
}

size_t wildcat_weights_workspace_size(int64_t BH, int64_t n, int d, int r) {
    if (BH < 0 || n < 1 || r < 1 || d < 1) return 0;
    return wildcat::weights_workspace_bytes(BH, n, d, r);
}

wildcat_status wildcat_weights(const float* F, const int32_t* S, const int32_t* rank, const void* V, int dtype,
                               int64_t BH, int64_t n, int d, int r, float* V_S, float* w, float* vmin, float* vmax,
                               void* workspace, size_t ws_bytes, void* stream) {
    const char* who = "wildcat_weights";
    wildcat_status st = check_common(dtype, BH, n, d, r, who);
    if (st != WILDCAT_OK) return st;
    if (BH == 0) return record(Status::ok());
    if (!F || !S || !rank || !V || !V_S || !w || !vmin || !vmax || !workspace)
        return bad(1, "%s: null pointer argument", who);
    if (!aligned16(V) || !aligned16(F)) return bad(1, "%s: F and V must be 16-byte aligned", who);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return bad(4, "%s: workspace must be 256-byte aligned", who);
    if (ws_bytes < wildcat::weights_workspace_bytes(BH, n, d, r)) return bad(4, "%s: workspace too small", who);
    wildcat::WeightsRequest q{F, S, rank, V, dtype, BH, n, d, r, V_S, w, vmin, vmax, workspace, ws_bytes};
    return record(wildcat::launch_weights(q, static_cast<cudaStream_t>(stream)));
}

size_t wildcat_weights_inverse_workspace_size(int64_t BH, int64_t n, int d, int r) {
    if (BH < 0 || n < 1 || r < 1 || d < 1 || r > wildcat::kInverseMaxRank) return 0;
    return wildcat::weights_inverse_workspace_bytes(BH, n, d, r);
}

wildcat_status wildcat_weights_inverse(const void* K, const void* V, int dtype, const int32_t* S,
                                       const int32_t* rank, int64_t BH, int64_t n, int d, int r, float beta,
                                       float* V_S, float* w, float* vmin, float* vmax, void* workspace,
                                       size_t ws_bytes, void* stream) {
    const char* who = "wildcat_weights_inverse";
    wildcat_status st = check_common(dtype, BH, n, d, r, who);
    if (st != WILDCAT_OK) return st;
    if ((st = check_scalars(beta, 0.f, who)) != WILDCAT_OK) return st;
    if (r > wildcat::kInverseMaxRank) return bad(2, "%s: r above 2048 is not supported", who);
    if (BH == 0) return record(Status::ok());
    if (!K || !V || !S || !rank || !V_S || !w || !vmin || !vmax || !workspace)
        return bad(1, "%s: null pointer argument", who);
    if (!aligned16(K) || !aligned16(V)) return bad(1, "%s: K and V must be 16-byte aligned", who);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return bad(4, "%s: workspace must be 256-byte aligned", who);
    if (ws_bytes < wildcat::weights_inverse_workspace_bytes(BH, n, d, r)) return bad(4, "%s: workspace too small", who);
    wildcat::WeightsInverseRequest q{K, V, dtype, S, rank, BH, n, d, r, beta, V_S, w, vmin, vmax, workspace, ws_bytes};
    return record(wildcat::launch_weights_inverse(q, static_cast<cudaStream_t>(stream)));
}

size_t wildcat_attend_workspace_size(int64_t BH, int64_t m, int d, int r) {
    if (BH < 0 || m < 0) return 0;
    return wildcat::attend_workspace_bytes(BH, m, d, r);
}

wildcat_status wildcat_attend(const void* Q, const void* K_S, int dtype, int64_t BH, int64_t m, int d, int r,
                              const int32_t* rank, float beta, const float* V_S, const float* w, const float* vmin,
                              const float* vmax, float* O, void* workspace, size_t ws_bytes, void* stream) {
    const char* who = "wildcat_attend";
    wildcat_status st = check_common(dtype, BH, r, d, r, who);
    if (st != WILDCAT_OK) return st;
    if ((st = check_scalars(beta, 0.f, who)) != WILDCAT_OK) return st;
    if (m < 0) return bad(1, "%s: m must be >= 0", who);
    if (BH == 0 || m == 0) return record(Status::ok());
    if (!Q || !K_S || !rank || !V_S || !w || !vmin || !vmax || !O || !workspace)
        return bad(1, "%s: null pointer argument", who);
    if (!aligned16(Q) || !aligned16(K_S)) return bad(1, "%s: Q and K_S must be 16-byte aligned", who);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return bad(4, "%s: workspace must be 256-byte aligned", who);
    if (ws_bytes < wildcat::attend_workspace_bytes(BH, m, d, r)) return bad(4, "%s: workspace too small", who);
    wildcat::AttendRequest q{Q, K_S, dtype, BH, m, d, r, rank, beta, V_S, w, vmin, vmax, O, workspace, ws_bytes};
    return record(wildcat::launch_attend(q, static_cast<cudaStream_t>(stream)));
}

wildcat_status wildcat_attend_noalloc(const void* Q, const void* K_S, int dtype, int64_t BH, int64_t m, int d, int r,
                                      const int32_t* rank, float beta, const float* V_S, const float* w,
                                      const float* vmin, const float* vmax, float* O, void* stream) {
    const char* who = "wildcat_attend_noalloc";
    wildcat_status st = check_common(dtype, BH, r, d, r, who);
    if (st != WILDCAT_OK) return st;
    if ((st = check_scalars(beta, 0.f, who)) != WILDCAT_OK) return st;
    if (m < 0) return bad(1, "%s: m must be >= 0", who);
    if (BH == 0 || m == 0) return record(Status::ok());
    if (!Q || !K_S || !rank || !V_S || !w || !vmin || !vmax || !O) return bad(1, "%s: null pointer argument", who);
    if (!aligned16(Q) || !aligned16(K_S)) return bad(1, "%s: Q and K_S must be 16-byte aligned", who);
    wildcat::AttendRequest q{Q, K_S, dtype, BH, m, d, r, rank, beta, V_S, w, vmin, vmax, O, nullptr, 0};
    return record(wildcat::launch_attend_noalloc(q, static_cast<cudaStream_t>(stream)));
}

size_t wildcat_decode_attend_workspace_size(int64_t BH, int d) {
    if (BH < 0 || d < 1) return 0;
    return wildcat::decode_workspace_bytes(BH, d);
}

wildcat_status wildcat_decode_attend(const void* Q_new, const void* K_new, const void* V_new, const void* K_S,
                                     int dtype, int64_t BH, int64_t m, int d, int r, const int32_t* rank, float beta,
                                     const float* V_S, const float* w, const float* vmin, const float* vmax, float* O,
                                     void* workspace, size_t ws_bytes, void* stream) {
    const char* who = "wildcat_decode_attend";
    wildcat_status st = check_common(dtype, BH, r, d, r, who);
    if (st != WILDCAT_OK) return st;
    if ((st = check_scalars(beta, 0.f, who)) != WILDCAT_OK) return st;
    if (m < 0) return bad(1, "%s: m must be >= 0", who);
    if (BH == 0 || m == 0) return record(Status::ok());
    if (!Q_new || !K_new || !V_new || !K_S || !rank || !V_S || !w || !vmin || !vmax || !O || !workspace)
        return bad(1, "%s: null pointer argument", who);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return bad(4, "%s: workspace must be 256-byte aligned", who);
    if (ws_bytes < wildcat::decode_workspace_bytes(BH, d)) return bad(4, "%s: workspace too small", who);
    wildcat::DecodeRequest q{Q_new, K_new, V_new, K_S, dtype, BH, m, d, r, rank, beta, V_S, w, vmin, vmax, O,
                             workspace, ws_bytes};
    return record(wildcat::launch_decode(q, static_cast<cudaStream_t>(stream)));
}

size_t wildcat_forward_workspace_size(int64_t BH, int64_t m, int64_t n, int d, int r, int dtype) {
    if (BH < 0 || m < 0 || n < 1 || r < 1 || d < 1) return 0;
    Carve cv(nullptr, 0);
    carve_forward(cv, BH, m, n, d, r, dtype);
    return cv.used + 256;
}

wildcat_status wildcat_forward(const void* Q, const void* K, const void* V, int dtype, int64_t BH, int64_t m,
                               int64_t n, int d, float beta, int r, uint64_t seed, int64_t inst0, float eps, float* O,
                               int32_t* S_out, int32_t* rank_out, void* workspace, size_t ws_bytes, void* stream) {
    const char* who = "wildcat_forward";
    wildcat_status st = check_common(dtype, BH, n, d, r, who);
    if (st != WILDCAT_OK) return st;
    if ((st = check_scalars(beta, eps, who)) != WILDCAT_OK) return st;
    if (m < 0) return bad(1, "%s: m must be >= 0", who);
    if (BH == 0) return record(Status::ok());
    if (!K || !V || !workspace || (m > 0 && (!Q || !O))) return bad(1, "%s: null pointer argument", who);
    if (!aligned16(K) || !aligned16(V) || (Q && !aligned16(Q)))
        return bad(1, "%s: Q, K and V must be 16-byte aligned", who);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return bad(4, "%s: workspace must be 256-byte aligned", who);
    Carve cv(workspace, ws_bytes);
    ForwardLayout L = carve_forward(cv, BH, m, n, d, r, dtype);
    if (!cv.fits()) return bad(4, "%s: workspace too small", who);
    if (inst0 < 0 || inst0 + BH > 4294967296LL) return bad(1, "%s: inst0 must satisfy 0 <= inst0, inst0 + BH <= 2^32", who);
    // the select writes the caller's pivot and rank arrays in place, and the
    // later stages read them from there (no copy at the end)
    if (S_out) L.S = S_out;
    if (rank_out) L.rank = rank_out;
    return forward_impl(Q, K, V, dtype, BH, m, n, d, beta, r, seed, inst0, eps, O, nullptr, nullptr, L,
                        static_cast<cudaStream_t>(stream));
}

size_t wildcat_forward_ex_workspace_size(int64_t BH, int64_t m, int64_t n, int d, int r, int dtype,
                                         const wildcat_options* opts) {
    const int nbins = opts ? opts->nbins : 1;
    if (BH < 0 || m < 0 || n < 1 || r < 1 || d < 1 || nbins < 1 || n % nbins || r % nbins) return 0;
    Carve cv(nullptr, 0);
    carve_binned(cv, BH, m, n, d, r, nbins, dtype, opts && opts->recenter);
    return cv.used + 256;
}

}  // extern "C"

namespace {

// Options of the extended forward, checked, with the key kernel's beta.
struct ExOptions {
    int nbins;
    bool recenter;
    float beta_key;  // beta / tau^2
};

wildcat_status check_ex(int dtype, int64_t BH, int64_t m, int64_t n, int d, float beta, int r, int64_t inst0, float eps,
                        const wildcat_options* opts, const char* who, ExOptions* out) {
    const int nbins = opts ? opts->nbins : 1;
    const float tau = opts ? opts->tau : 1.f;
    wildcat_status st = check_common(dtype, BH, n, d, r, who);
    if (st != WILDCAT_OK) return st;
    if ((st = check_scalars(beta, eps, who)) != WILDCAT_OK) return st;
    if ((st = check_bins(BH, n, r, nbins, who)) != WILDCAT_OK) return st;
    if (opts && opts->recenter != 0 && opts->recenter != 1) return bad(1, "%s: recenter must be 0 or 1", who);
    if (!std::isfinite(tau) || !(tau > 0.f)) return bad(1, "%s: tau must be finite and > 0", who);
    const float beta_key = beta / (tau * tau);
    if (!std::isfinite(beta_key) || !(beta_key > 0.f)) return bad(1, "%s: beta / tau^2 must be finite and > 0", who);
    if (m < 0) return bad(1, "%s: m must be >= 0", who);
    if (inst0 < 0 || (inst0 + BH) * nbins > 4294967296LL)
        return bad(1, "%s: inst0 must satisfy 0 <= inst0, (inst0 + BH) * nbins <= 2^32", who);
    *out = ExOptions{nbins, opts && opts->recenter, beta_key};
    return WILDCAT_OK;
}

// The extended forward on device buffers: recentring mean, select and weights
// on the [BH * nbins, n / nbins] view, the bins' union coreset, attend.
// wait_v / wait_q (optional): events the weights / attend stage waits for.
wildcat_status forward_ex_impl(const void* Q, const void* K, const void* V, int dtype, int64_t BH, int64_t m, int64_t n,
                               int d, float beta, int r, uint64_t seed, int64_t inst0, float eps, const ExOptions& o,
                               float* O, int32_t* S_out, int32_t* rank_out, const BinnedLayout& L, cudaStream_t s,
                               cudaEvent_t wait_v = nullptr, cudaEvent_t wait_q = nullptr) {
    const int nbins = o.nbins;
    const int64_t nb = n / nbins, BB = BH * nbins;
    const int rb = r / nbins;
    Status z;
    cudaError_t ew;
    std::unique_lock<std::mutex> aux_lock;
    AuxPipe* ap = nullptr;
    bool forked = false;
    if ((z = fork_value_range(V, dtype, BB, nb, d, L.vmin_b, L.vmax_b, L.rws, L.rws_bytes, s, wait_v, aux_lock, &ap,
                              &forked)).code)
        return record(z);
    if (o.recenter && (z = wildcat::launch_key_mean(K, dtype, BH, n, d, L.mws, L.kbar, s)).code) return record(z);
    wildcat::SelectRequest sq{K,      dtype, BB,      nb,  d,     o.beta_key, rb,      seed, inst0 * nbins,
                              eps,    nullptr, L.S,   L.F, L.rank_b, L.K_S,   L.kbar,  nbins};
    sq.ws = L.sws;
    sq.ws_bytes = L.sws_bytes;
    if ((z = wildcat::launch_select(sq, s)).code) return record(z);
    if ((z = mark_stage(g_ev_after_select, s, "forward: stage event")).code) return record(z);
    if (wait_v && (ew = cudaStreamWaitEvent(s, wait_v, 0))) return record(Status::cuda(ew, "forward: wait for V"));
    wildcat::WeightsRequest wq{L.F, L.S, L.rank_b, V, dtype, BB, nb, d, rb, L.V_S, L.w, L.vmin_b, L.vmax_b, L.wws,
                               L.wws_bytes};
    wq.skip_range = forked;
    if ((z = wildcat::launch_weights(wq, s)).code) return record(z);
    if ((z = mark_stage(g_ev_after_weights, s, "forward: stage event")).code) return record(z);
    if (forked && (z = join_value_range(ap, s, aux_lock)).code) return record(z);
    if ((z = wildcat::launch_binning_finish(L.vmin_b, L.vmax_b, L.S, L.rank_b, BH, nbins, nb, rb, d, L.vmin, L.vmax,
                                            L.rank_att, S_out, rank_out, s)).code)
        return record(z);
    if (wait_q && (ew = cudaStreamWaitEvent(s, wait_q, 0))) return record(Status::cuda(ew, "forward: wait for Q"));
    if (m > 0) {
        // the attend is unchanged by recentring and temperature: it uses the
        // original pivot keys and beta (the shift and 1/tau cancel in N / D)
        wildcat::AttendRequest aq{Q,      L.K_S,  dtype, BH, m, d, r, L.rank_att, beta, L.V_S, L.w,
                                  L.vmin, L.vmax, O,     L.aws, L.aws_bytes};
        if ((z = wildcat::launch_attend(aq, s)).code) return record(z);
    }
    return record(Status::ok());
}

}  // namespace

extern "C" {

wildcat_status wildcat_forward_ex(const void* Q, const void* K, const void* V, int dtype, int64_t BH, int64_t m,
                                  int64_t n, int d, float beta, int r, uint64_t seed, int64_t inst0, float eps,
                                  const wildcat_options* opts, float* O, int32_t* S_out, int32_t* rank_out,
                                  void* workspace, size_t ws_bytes, void* stream) {
    const char* who = "wildcat_forward_ex";
    ExOptions o{};
    wildcat_status st = check_ex(dtype, BH, m, n, d, beta, r, inst0, eps, opts, who, &o);
    if (st != WILDCAT_OK) return st;
    if (BH == 0) return record(Status::ok());
    if (!K || !V || !workspace || (m > 0 && (!Q || !O))) return bad(1, "%s: null pointer argument", who);
    if (!aligned16(K) || !aligned16(V) || (Q && !aligned16(Q)))
        return bad(1, "%s: Q, K and V must be 16-byte aligned", who);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return bad(4, "%s: workspace must be 256-byte aligned", who);
    Carve cv(workspace, ws_bytes);
    const BinnedLayout L = carve_binned(cv, BH, m, n, d, r, o.nbins, dtype, o.recenter);
    if (!cv.fits()) return bad(4, "%s: workspace too small", who);
    return forward_ex_impl(Q, K, V, dtype, BH, m, n, d, beta, r, seed, inst0, eps, o, O, S_out, rank_out, L,
                           static_cast<cudaStream_t>(stream));
}

size_t wildcat_forward_binned_workspace_size(int64_t BH, int64_t m, int64_t n, int d, int r, int nbins, int dtype) {
    const wildcat_options o{nbins, 0, 1.f};
    return wildcat_forward_ex_workspace_size(BH, m, n, d, r, dtype, &o);
}

wildcat_status wildcat_forward_binned(const void* Q, const void* K, const void* V, int dtype, int64_t BH, int64_t m,
                                      int64_t n, int d, float beta, int r, int nbins, uint64_t seed, int64_t inst0,
                                      float eps, float* O, int32_t* S_out, int32_t* rank_out, void* workspace,
                                      size_t ws_bytes, void* stream) {
    const wildcat_options o{nbins, 0, 1.f};
    return wildcat_forward_ex(Q, K, V, dtype, BH, m, n, d, beta, r, seed, inst0, eps, &o, O, S_out, rank_out,
                              workspace, ws_bytes, stream);
}

size_t wildcat_forward_host_workspace_size(int64_t BH, int64_t m, int64_t n, int d, int r, int dtype) {
    if (BH < 0 || m < 0 || n < 1 || r < 1 || d < 1) return 0;
    Carve cv(nullptr, 0);
    cv.take(elem_bytes(dtype) * BH * m * d);
    cv.take(elem_bytes(dtype) * BH * n * d);
    cv.take(elem_bytes(dtype) * BH * n * d);
    cv.take(sizeof(float) * BH * m * d);
    cv.take(sizeof(int32_t) * BH * r);
    cv.take(sizeof(int32_t) * BH);
    carve_forward(cv, BH, m, n, d, r, dtype);
    return cv.used + 256;
}

wildcat_status wildcat_forward_host(const void* Q_host, const void* K_host, const void* V_host, int dtype, int64_t BH,
                                    int64_t m, int64_t n, int d, float beta, int r, uint64_t seed, int64_t inst0,
                                    float eps, float* O_host, int32_t* S_host, int32_t* rank_host, void* workspace,
                                    size_t ws_bytes, void* stream) {
    const char* who = "wildcat_forward_host";
    wildcat_status st = check_common(dtype, BH, n, d, r, who);
    if (st != WILDCAT_OK) return st;
    if ((st = check_scalars(beta, eps, who)) != WILDCAT_OK) return st;
    if (m < 0) return bad(1, "%s: m must be >= 0", who);
    if (BH == 0) return record(Status::ok());
    if (!K_host || !V_host || !workspace || (m > 0 && (!Q_host || !O_host)))
        return bad(1, "%s: null pointer argument", who);
    if (inst0 < 0 || inst0 + BH > 4294967296LL) return bad(1, "%s: inst0 must satisfy 0 <= inst0, inst0 + BH <= 2^32", who);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return bad(4, "%s: workspace must be 256-byte aligned", who);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t eb = elem_bytes(dtype);
    Carve cv(workspace, ws_bytes);
    void* Qd = cv.take(eb * BH * m * d);
    void* Kd = cv.take(eb * BH * n * d);
    void* Vd = cv.take(eb * BH * n * d);
    float* Od = static_cast<float*>(cv.take(sizeof(float) * BH * m * d));
    cv.take(sizeof(int32_t) * BH * r);
    cv.take(sizeof(int32_t) * BH);
    const ForwardLayout L = carve_forward(cv, BH, m, n, d, r, dtype);
    if (!cv.fits()) return bad(4, "%s: workspace too small", who);
    // K first on a copy stream: the select needs only K, so V and Q cross
    // the bus while it runs; the weights and attend stages wait for them.
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e) return record(Status::cuda(e, "forward_host: current device"));
    HostPipe* hp = host_pipe(dev);
    if (!hp) return record(Status::cuda(cudaErrorMemoryAllocation, "forward_host: copy stream"));
    std::lock_guard<std::mutex> lock(hp->mu);
    Status z = stage_host_inputs(hp, s, Kd, Vd, Qd, K_host, V_host, Q_host, eb * BH * n * d, eb * BH * m * d);
    if (z.code) {
        cudaStreamSynchronize(hp->cs);
        return record(z);
    }
    st = forward_impl(m > 0 ? Qd : nullptr, Kd, Vd, dtype, BH, m, n, d, beta, r, seed, inst0, eps,
                      m > 0 ? Od : nullptr, nullptr, nullptr, L, s, hp->v_in, hp->q_in);
    if (st != WILDCAT_OK) {
        cudaStreamSynchronize(hp->cs);
        return st;
    }
    if (m > 0 && (e = cudaMemcpyAsync(O_host, Od, sizeof(float) * BH * m * d, cudaMemcpyDeviceToHost, s)))
        return record(Status::cuda(e, "forward_host: copy O"));
    if (S_host && (e = cudaMemcpyAsync(S_host, L.S, sizeof(int32_t) * BH * r, cudaMemcpyDeviceToHost, s)))
        return record(Status::cuda(e, "forward_host: copy S"));
    if (rank_host && (e = cudaMemcpyAsync(rank_host, L.rank, sizeof(int32_t) * BH, cudaMemcpyDeviceToHost, s)))
        return record(Status::cuda(e, "forward_host: copy rank"));
    if ((e = cudaStreamSynchronize(s))) return record(Status::cuda(e, "forward_host: stream sync"));
    return record(Status::ok());
}

size_t wildcat_forward_ex_host_workspace_size(int64_t BH, int64_t m, int64_t n, int d, int r, int dtype,
                                              const wildcat_options* opts) {
    const int nbins = opts ? opts->nbins : 1;
    if (BH < 0 || m < 0 || n < 1 || r < 1 || d < 1 || nbins < 1 || n % nbins || r % nbins) return 0;
    Carve cv(nullptr, 0);
    cv.take(elem_bytes(dtype) * BH * m * d);
    cv.take(elem_bytes(dtype) * BH * n * d);
    cv.take(elem_bytes(dtype) * BH * n * d);
    cv.take(sizeof(float) * BH * m * d);
    cv.take(sizeof(int32_t) * BH * r);
    cv.take(sizeof(int32_t) * BH * nbins);
    carve_binned(cv, BH, m, n, d, r, nbins, dtype, opts && opts->recenter);
    return cv.used + 256;
}

wildcat_status wildcat_forward_ex_host(const void* Q_host, const void* K_host, const void* V_host, int dtype,
                                       int64_t BH, int64_t m, int64_t n, int d, float beta, int r, uint64_t seed,
                                       int64_t inst0, float eps, const wildcat_options* opts, float* O_host,
                                       int32_t* S_host, int32_t* rank_host, void* workspace, size_t ws_bytes,
                                       void* stream) {
    const char* who = "wildcat_forward_ex_host";
    ExOptions o{};
    wildcat_status st = check_ex(dtype, BH, m, n, d, beta, r, inst0, eps, opts, who, &o);
    if (st != WILDCAT_OK) return st;
    if (BH == 0) return record(Status::ok());
    if (!K_host || !V_host || !workspace || (m > 0 && (!Q_host || !O_host)))
        return bad(1, "%s: null pointer argument", who);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return bad(4, "%s: workspace must be 256-byte aligned", who);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t eb = elem_bytes(dtype);
    Carve cv(workspace, ws_bytes);
    void* Qd = cv.take(eb * BH * m * d);
    void* Kd = cv.take(eb * BH * n * d);
    void* Vd = cv.take(eb * BH * n * d);
    float* Od = static_cast<float*>(cv.take(sizeof(float) * BH * m * d));
    int32_t* Sd = static_cast<int32_t*>(cv.take(sizeof(int32_t) * BH * r));
    int32_t* rankd = static_cast<int32_t*>(cv.take(sizeof(int32_t) * BH * o.nbins));
    const BinnedLayout L = carve_binned(cv, BH, m, n, d, r, o.nbins, dtype, o.recenter);
    if (!cv.fits()) return bad(4, "%s: workspace too small", who);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e) return record(Status::cuda(e, "forward_host: current device"));
    HostPipe* hp = host_pipe(dev);
    if (!hp) return record(Status::cuda(cudaErrorMemoryAllocation, "forward_host: copy stream"));
    std::lock_guard<std::mutex> lock(hp->mu);
    Status z = stage_host_inputs(hp, s, Kd, Vd, Qd, K_host, V_host, Q_host, eb * BH * n * d, eb * BH * m * d);
    if (z.code) {
        cudaStreamSynchronize(hp->cs);
        return record(z);
    }
    st = forward_ex_impl(m > 0 ? Qd : nullptr, Kd, Vd, dtype, BH, m, n, d, beta, r, seed, inst0, eps, o,
                         m > 0 ? Od : nullptr, Sd, rankd, L, s, hp->v_in, hp->q_in);
    if (st != WILDCAT_OK) {
        cudaStreamSynchronize(hp->cs);
        return st;
    }
    if (m > 0 && (e = cudaMemcpyAsync(O_host, Od, sizeof(float) * BH * m * d, cudaMemcpyDeviceToHost, s)))
        return record(Status::cuda(e, "forward_host: copy O"));
    if (S_host && (e = cudaMemcpyAsync(S_host, Sd, sizeof(int32_t) * BH * r, cudaMemcpyDeviceToHost, s)))
        return record(Status::cuda(e, "forward_host: copy S"));
    if (rank_host && (e = cudaMemcpyAsync(rank_host, rankd, sizeof(int32_t) * BH * o.nbins, cudaMemcpyDeviceToHost, s)))
        return record(Status::cuda(e, "forward_host: copy rank"));
    if ((e = cudaStreamSynchronize(s))) return record(Status::cuda(e, "forward_host: stream sync"));
    return record(Status::ok());
}

wildcat_status wildcat_pivot_uniforms(uint64_t seed, int64_t BH, int steps, double* u, void* stream) {
    if (BH < 0 || steps < 0) return bad(1, "%s: BH and steps must be >= 0", "wildcat_pivot_uniforms");
    if (BH * (int64_t)steps > 0 && !u) return bad(1, "%s: u must be non-null", "wildcat_pivot_uniforms");
    return record(wildcat::launch_pivot_uniforms(seed, BH, steps, u, static_cast<cudaStream_t>(stream)));
}

wildcat_status wildcat_get_device_status(void* stream) {
    const cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return record(Status::cuda(e, "wildcat_get_device_status: stream sync"));
    const int v = wildcat::read_device_status(true);
    if (v < 0) return record(Status::fail(3, "wildcat_get_device_status: cannot read the status word"));
    if (v == WILDCAT_ERR_TIMEOUT) return record(Status::fail(5, "a kernel's bounded wait expired"));
    return record(Status::ok());
}

wildcat_status wildcat_test_force_wait_timeout(int64_t nanoseconds) {
    if (nanoseconds < 0 || nanoseconds > 1000000000LL)
        return bad(1, "%s: nanoseconds must be in [0, 1e9]", "wildcat_test_force_wait_timeout");
    wildcat::set_attend_force_timeout((unsigned long long)nanoseconds);
    return record(Status::ok());
}

wildcat_status wildcat_test_force_select_timeout(int64_t nanoseconds) {
    if (nanoseconds < 0 || nanoseconds > 1000000000LL)
        return bad(1, "%s: nanoseconds must be in [0, 1e9]", "wildcat_test_force_select_timeout");
    wildcat::set_select_force_timeout((unsigned long long)nanoseconds);
    return record(Status::ok());
}

wildcat_status wildcat_set_select_kernel(int kernel) {
    if (kernel != 0 && kernel != 1 && kernel != 3)
        return bad(1, "%s: kernel must be 0 (automatic), 1 (clusters) or 3 (global sync)",
                   "wildcat_set_select_kernel");
    wildcat::select_kernel_override(kernel);
    return record(Status::ok());
}

int wildcat_last_select_kernel(void) { return wildcat::last_select_kernel(); }

int wildcat_last_select_threads(void) { return wildcat::last_select_threads(); }

wildcat_status wildcat_set_select_phase_steps(int steps) {
    wildcat::select_phase_steps_override(steps, true);
    return record(Status::ok());
}

int wildcat_last_select_phases(void) { return wildcat::last_select_phases(); }

wildcat_status wildcat_set_stage_events(void* after_select, void* after_weights) {
    g_ev_after_select = static_cast<cudaEvent_t>(after_select);
    g_ev_after_weights = static_cast<cudaEvent_t>(after_weights);
    return record(Status::ok());
}

wildcat_status wildcat_set_select_cluster(int ctas_per_instance) {
    const int G = ctas_per_instance;
    if (G != 0 && G != 1 && G != 2 && G != 4 && G != 8 && G != 16)
        return bad(1, "%s: cluster size must be 0 (auto) or a power of two <= 16", "wildcat_set_select_cluster");
    wildcat::select_cluster_override(G);
    return record(Status::ok());
}

int wildcat_last_select_cluster(void) { return wildcat::last_select_cluster(); }

}  // extern "C"
