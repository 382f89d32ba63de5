// Planner and executor of one Muon call: shape groups, workspace layout, the
// Newton-Schulz op chain of each group, and its lowering into grouped kernel
// launches (tensor-core or fp32 SIMT).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <string>
#include <vector>

#include "launch.h"
#include "muon_internal.h"

namespace muon {

enum NsForm { FORM_STANDARD = 0, FORM_GRAM = 1, FORM_AUTO = 2 };

// What one call asks for.  Matrices are in the caller's layout (rows x cols).
struct PlanRequest {
    // matrices
    std::vector<int> rows, cols;
    std::vector<const void*> in;   // gradients (step) or inputs (orthogonalize)
    std::vector<void*> mom;        // momentum buffers (step) or empty
    std::vector<void*> out;        // params (step) or outputs (orthogonalize, == in)
    int in_dt = DT_BF16;           // dtype of `in`
    int mom_dt = DT_BF16;
    int out_dt = DT_BF16;          // dtype of `out`
    bool is_step = false;          // W -= lr*O (else out = O)
    bool fp32_path = false;        // fp32 SIMT check path (orthogonalize only)
    int form = FORM_AUTO;
    int steps = 5;
    std::vector<float> coeffs;     // 3*steps
    // Per-shape schedules: matrix i uses scheds[sched[i]] when sched is not
    // empty and sched[i] >= 0, else (steps, coeffs) above.
    struct Schedule {
        int steps = 0;
        std::vector<float> coeffs;  // 3*steps
    };
    std::vector<Schedule> scheds;
    std::vector<int> sched;
    unsigned restart_mask = 1u << 2;
    float eps = 1e-7f;
    float mu = 0.95f;
    int nesterov = 1;
    float lr = 0.f;
    float clip = 0.f;              // muon_step: the update is clipped to [-clip, clip] (0 = off)
    int device = 0;
    int index_base = 0;            // caller's index of matrix 0 (status reporting; per call, not in the key)
};

struct LaunchRec {
    enum Kind { MOM, TC, F32, SCALE } kind;
    TcLaunch tc{};
    int grid = 0;
    F32Launch f32{};
    MomLaunch mom{};
    ScaleLaunch sc{};
    double flops = 0, bytes = 0;
    double extra_bytes = 0;  // the AdamW lane of a hybrid step (momentum launch)
    char label[32] = {};     // NVTX range name of the launch (phase and chain slot)
};

struct ProfileSink {
    virtual void before(cudaStream_t s) = 0;
    virtual void after(cudaStream_t s, int kind, double flops, double bytes) = 0;
    virtual ~ProfileSink() = default;
};

class Plan {
  public:
    // Build a plan (host tables + device workspace).  Returns a MUON_* status
    // and fills err on failure.
    int build(const PlanRequest& req, DeviceStatus* status, int num_sms, cudaStream_t stream, std::string& err);
    // True when `req` differs from the built plan only in mu, nesterov, lr.
    bool same_shape_key(const PlanRequest& req) const;
    // Patch the per-call scalars (mu, nesterov, lr) into the launch records.
    void set_scalars(float mu, int nesterov, float lr, float clip);
    // Patch the caller's index of matrix 0 (the first non-finite matrix is
    // reported in the caller's numbering).
    void set_index_base(int base);
    // Append (or, with null, remove) an AdamW lane to the momentum launch's
    // grid; `bytes` are its algorithmic HBM bytes (tracing).
    void set_adamw(const AdamLaunch* adam, double bytes);
    int run(cudaStream_t stream, ProfileSink* prof, long long* launch_counter, std::string& err);
    void release();
    ~Plan() { release(); }
    // Debug canary mode: the workspace guards (none when the mode is off).
    int guard_count() const { return static_cast<int>(guard_offs_.size()); }
    void* guard_addr(int i) const { return static_cast<char*>(arena_) + guard_offs_[static_cast<size_t>(i)]; }

    std::vector<LaunchRec> launches;
    size_t arena_bytes = 0;
    double total_flops = 0;

  private:
    std::vector<long long> key_;
    void* arena_ = nullptr;
    bool fault_launch_ = false;  // MUON_FAULT=launch: run() fails before its first launch
    // MUON_DEBUG_CANARY=1: offsets of the guard after every workspace region,
    // their device copy, and the status word the check reports to
    std::vector<unsigned long long> guard_offs_;
    const unsigned long long* d_guard_offs_ = nullptr;
    DeviceStatus* status_ = nullptr;
};

// Exposed for tests of the host logic: algorithmic FLOPs of one matrix.
double ns_flops(int n, int m, int steps, int form, unsigned restart_mask);
// Form chosen for an n x m (n <= m) matrix under `form` (AUTO resolves here).
int resolve_form(int n, int m, int steps, int form, unsigned restart_mask);

}  // namespace muon
