// internal.h -- host-side interfaces between the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace wildcat {

// Result of a host-side launcher: code follows wildcat_status.
struct Status {
    int code;
    const char* what;      // static text
    cudaError_t cuda_err;  // for code 3
    static Status ok() { return {0, "", cudaSuccess}; }
    static Status fail(int c, const char* w) { return {c, w, cudaSuccess}; }
    static Status cuda(cudaError_t e, const char* w) { return {3, w, e}; }
};

struct SelectRequest {
    const void* K;
    int dtype;  // 0 f32, 1 bf16
    int64_t BH, n;
    int d;
    float beta;
    int r;
    uint64_t seed;
    int64_t inst0;
    float eps;
    const int32_t* S_fixed;
    int32_t* S;
    float* F;
    int32_t* rank;
    void* K_S;
    const float* kbar = nullptr;  // recentring: per-instance key mean (or nullptr)
    int kbar_div = 1;             // instance b uses kbar row b / kbar_div
    void* ws = nullptr;           // optional workspace (global-sync mode), 256-byte aligned
    size_t ws_bytes = 0;
};

Status launch_select(const SelectRequest& q, cudaStream_t stream);
Status launch_pivot_uniforms(uint64_t seed, int64_t BH, int steps, double* u, cudaStream_t stream);
int select_cluster_override(int G);  // G < 0: query only
int last_select_cluster();
int select_kernel_override(int k);  // k < 0: query only; 0 automatic, 1 clusters, 3 global sync where a
                                    // workspace allows
int last_select_kernel();           // 1 clusters, 3 global sync
int last_select_threads();          // threads per CTA of the last select launch (256 or 512)
int select_phase_steps_override(int k, bool set);  // steps per launch: 0 automatic, < 0 one launch
int last_select_phases();           // launches of the last select call (1 = no phases)
// cluster-size choice of the select kernel (select.cu)
struct ClusterKey {
    int dev, kernel;
    int64_t n, BH;
    int r, d, dtype;
    bool operator<(const ClusterKey& o) const;
};
int cached_cluster_lookup(const ClusterKey& key);   // 0 if absent
void cached_cluster_store(const ClusterKey& key, int G);
int choose_cluster_rows(int64_t n, int64_t BH, int (*fit)(int G, void* ctx), void* ctx, double* cost_out,
                        int min_rows = 512);
size_t select_workspace_bytes(int64_t BH, int64_t n);  // global-sync exchange buffers
int read_select_gs_status(bool clear);
// test hook: the global-sync barrier of the select waits on a counter that
// one CTA never bumps for `ns` nanoseconds (0 = off)
void set_select_force_timeout(unsigned long long ns);
unsigned long long select_force_timeout_ns();

// ---- weights: Y = F^T (V, 1), then F_S^T X = Y ----
struct WeightsRequest {
    const float* F;
    const int32_t* S;
    const int32_t* rank;
    const void* V;
    int dtype;
    int64_t BH, n;
    int d, r;
    float* V_S;
    float* w;
    float* vmin;
    float* vmax;
    void* ws;
    size_t ws_bytes;
    bool skip_range = false;  // vmin / vmax are formed elsewhere (launch_value_range)
};
size_t weights_workspace_bytes(int64_t BH, int64_t n, int d, int r);
Status launch_weights(const WeightsRequest& q, cudaStream_t stream);
// column-wise value range of V alone (the same kernels as launch_weights)
size_t value_range_workspace_bytes(int64_t BH, int64_t n, int d);
Status launch_value_range(const void* V, int dtype, int64_t BH, int64_t n, int d, float* vmin, float* vmax,
                          void* ws, size_t ws_bytes, cudaStream_t stream);
// weights through the maintained inverse of h(K_S, K_S) (weights_inverse.cu)
struct WeightsInverseRequest {
    const void* K;
    const void* V;
    int dtype;
    const int32_t* S;
    const int32_t* rank;
    int64_t BH, n;
    int d, r;
    float beta;
    float* V_S;
    float* w;
    float* vmin;
    float* vmax;
    void* ws;
    size_t ws_bytes;
};
size_t weights_inverse_workspace_bytes(int64_t BH, int64_t n, int d, int r);
Status launch_weights_inverse(const WeightsInverseRequest& q, cudaStream_t stream);
constexpr int kInverseMaxRank = 2048;
// tensor-core F^T (V, 1) partials (weights_tc.cu)
bool weights_tc_supported(int dtype, int d, int64_t n);
int64_t weights_tc_keys_per_split(int64_t BH, int64_t n, int d, int r, int sms);
Status launch_weights_tc(const float* F, const void* V, const int32_t* rank, int64_t BH, int64_t n, int d, int r,
                         int nsplit, int64_t keys_per_split, float* Ypart, cudaStream_t stream);

// ---- attend ----
struct AttendRequest {
    const void* Q;
    const void* K_S;
    int dtype;
    int64_t BH, m;
    int d, r;
    const int32_t* rank;
    float beta;
    const float* V_S;
    const float* w;
    const float* vmin;
    const float* vmax;
    float* O;
    void* ws;
    size_t ws_bytes;
};
size_t attend_workspace_bytes(int64_t BH, int64_t m, int d, int r);
size_t attend_simt_workspace_bytes(int64_t BH, int64_t m);
Status launch_attend(const AttendRequest& q, cudaStream_t stream);
Status launch_attend_simt(const AttendRequest& q, cudaStream_t stream);
// tensor-core attend (attend_tc.cu)
bool attend_tc_supported(int dtype, int d);
size_t attend_tc_scratch_bytes(int64_t BH, int d, int r);
Status launch_attend_tc(const AttendRequest& q, void* scratch, cudaStream_t stream);
// device status word set by bounded waits that expired (0 = none); -1 if unreadable
int read_device_status(bool clear);  // first non-zero of the per-file status words below
int read_attend_status(bool clear);
int read_weights_status(bool clear);
// test hook: the tensor-core attend first waits `ns` nanoseconds on a barrier
// that nothing completes, then reports a timeout (0 = off)
void set_attend_force_timeout(unsigned long long ns);
// attend with its scratch in a static device array (no workspace argument)
size_t attend_noalloc_scratch_bytes();
Status launch_attend_noalloc(const AttendRequest& q, cudaStream_t stream);

// KV-cache decode with new tokens (decode.cu)
struct DecodeRequest {
    const void* Qn;
    const void* Kn;
    const void* Vn;
    const void* K_S;
    int dtype;
    int64_t BH, m;
    int d, r;
    const int32_t* rank;
    float beta;
    const float* V_S;
    const float* w;
    const float* vmin;
    const float* vmax;
    float* O;
    void* ws;
    size_t ws_bytes;
};
size_t decode_workspace_bytes(int64_t BH, int d);
Status launch_decode(const DecodeRequest& q, cudaStream_t stream);

// per-instance key mean (binning.cu), fp64 partial sums then fp32 mean
size_t key_mean_workspace_bytes(int64_t BH, int64_t n, int d);
Status launch_key_mean(const void* K, int dtype, int64_t BH, int64_t n, int d, void* ws, float* kbar,
                       cudaStream_t st);

// binned forward glue (binning.cu)
Status launch_binning_finish(const float* vmin_b, const float* vmax_b, const int32_t* S_b, const int32_t* rank_b,
                             int64_t BH, int nbins, int64_t nb, int rb, int d, float* vmin, float* vmax,
                             int32_t* rank_att, int32_t* S_out, int32_t* rank_out, cudaStream_t st);

// 256-byte aligned bump allocator over a caller-provided workspace.
struct Carve {
    char* base;
    size_t cap, used;
    explicit Carve(void* p, size_t c) : base(static_cast<char*>(p)), cap(c), used(0) {}
    void* take(size_t bytes) {
        const size_t at = (used + 255) & ~size_t(255);
        used = at + bytes;
        return base ? base + at : nullptr;
    }
    bool fits() const { return used <= cap; }
};

}  // namespace wildcat
