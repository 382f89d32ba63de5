// C ABI of the Muon library (include/muon.h): argument validation, config,
// stream binding, the device status word, tracing, and the two entry points.
// No exception crosses this boundary; every entry point returns a status.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <deque>
#include <memory>
#include <string>
#include <vector>

#include "../../include/muon.h"
#include "plan.h"

using namespace muon;

namespace {

thread_local std::string g_err;
muon_config g_cfg;
bool g_cfg_init = false;
cudaStream_t g_stream = nullptr;
std::atomic<long long> g_launches{0};

struct DeviceState {
    int device = -1;
    int num_sms = 0;
    int cc_major = 0, cc_minor = 0;
    DeviceStatus* status = nullptr;
    std::unique_ptr<Plan> plan;
    void* adam_table = nullptr;  // AdamW tensor table
    size_t adam_cap = 0;
    std::vector<AdamTensor> adam_last;  // contents of adam_table
    // The workspace (plan tables, intermediates, AdamW table) is reused by
    // every call.  ws_event marks the end of its last use, on ws_stream; a
    // call on another stream first makes its stream wait for that event, so
    // its table uploads and kernels cannot overlap the previous call's.
    cudaEvent_t ws_event = nullptr;
    cudaStream_t ws_stream = nullptr;
    bool ws_used = false;
    // muon_step_offload: one cached plan per group of matrices (the groups
    // run back to back on the bound stream, so none rebuilds another's), and
    // the two copy streams with their events (created on first use)
    std::vector<std::unique_ptr<Plan>> chunk_plans;
    cudaStream_t copy_in = nullptr, copy_out = nullptr;
    cudaEvent_t ev_start = nullptr, ev_out = nullptr;
    std::vector<cudaEvent_t> ev_in, ev_done;  // per group: gradients landed, group stepped
};
std::deque<DeviceState> g_devs;  // deque: references stay valid on growth

// Per-shape Newton-Schulz schedules of muon_step, keyed by the short and the
// long side of the matrix.
struct ShapeSchedule {
    int n, m, steps;
    std::vector<float> coeffs;
};
std::vector<ShapeSchedule> g_shape_scheds;

int fail(int code, const std::string& msg) {
    g_err = msg;
    return code;
}

// Defaults: five steps of the tuned quintic (3.4445, -4.7750, 2.0315)
// ([NanoGPT-Muon] "Newton-Schulz 迭代的系数调优"), per-matrix choice of the
// cheaper form, one Gram restart before step 2, eps 1e-7, bf16 momentum,
// fp32 parameters.
void fill_defaults(muon_config* c) {
    std::memset(c, 0, sizeof(*c));
    c->steps = 5;
    for (int k = 0; k < MUON_MAX_STEPS; ++k) {
        c->coeffs[3 * k] = 3.4445f;
        c->coeffs[3 * k + 1] = -4.7750f;
        c->coeffs[3 * k + 2] = 2.0315f;
    }
    c->mode = MUON_NS_AUTO;
    c->restart_mask = 1u << 2;
    c->eps = 1e-7f;
    c->momentum_dtype = MUON_DTYPE_BF16;
    c->param_dtype = MUON_DTYPE_F32;
    c->grad_dtype = MUON_DTYPE_BF16;
    c->soft_threshold = 0.f;
}

void ensure_cfg() {
    if (g_cfg_init) return;
    fill_defaults(&g_cfg);
    g_cfg_init = true;
}

int check_cfg(const muon_config& c) {
    if (c.steps < 0 || c.steps > MUON_MAX_STEPS) return fail(MUON_ERR_INVALID_ARG, "config.steps out of range");
    if ((c.mode & ~MUON_NS_FORM_MASK) != 0 || c.mode < 0 || c.mode > MUON_NS_AUTO)
        return fail(MUON_ERR_INVALID_ARG, "config.mode must be MUON_NS_STANDARD, MUON_NS_GRAM or MUON_NS_AUTO");
    if (!(c.eps >= 0.f) || !std::isfinite(c.eps)) return fail(MUON_ERR_INVALID_ARG, "config.eps must be finite and >= 0");
    for (int i = 0; i < 3 * c.steps; ++i)
        if (!std::isfinite(c.coeffs[i])) return fail(MUON_ERR_INVALID_ARG, "config.coeffs must be finite");
    if (c.momentum_dtype != MUON_DTYPE_BF16 && c.momentum_dtype != MUON_DTYPE_F32)
        return fail(MUON_ERR_UNSUPPORTED, "config.momentum_dtype must be BF16 or F32");
    if (c.param_dtype != MUON_DTYPE_BF16 && c.param_dtype != MUON_DTYPE_F32)
        return fail(MUON_ERR_UNSUPPORTED, "config.param_dtype must be BF16 or F32");
    if (c.grad_dtype != MUON_DTYPE_BF16 && c.grad_dtype != MUON_DTYPE_F32)
        return fail(MUON_ERR_UNSUPPORTED, "config.grad_dtype must be BF16 or F32");
    if (!std::isfinite(c.soft_threshold) || c.soft_threshold < 0.f)
        return fail(MUON_ERR_INVALID_ARG, "config.soft_threshold must be finite and >= 0");
    return MUON_OK;
}

// Current device's state; allocates the status word on first use.
int device_state(DeviceState** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(MUON_ERR_CUDA, std::string("no CUDA device: ") + cudaGetErrorString(e));
    }
    for (DeviceState& d : g_devs)
        if (d.device == dev) {
            *out = &d;
            return MUON_OK;
        }
    DeviceState d;
    d.device = dev;
    cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (cudaMalloc(&d.status, sizeof(DeviceStatus)) != cudaSuccess) {
        cudaGetLastError();
        return fail(MUON_ERR_NO_MEMORY, "status word allocation failed");
    }
    const DeviceStatus init{0, 0x7fffffff};
    cudaMemcpy(d.status, &init, sizeof(init), cudaMemcpyHostToDevice);
    if (cudaEventCreateWithFlags(&d.ws_event, cudaEventDisableTiming) != cudaSuccess) {
        cudaGetLastError();
        cudaFree(d.status);
        return fail(MUON_ERR_CUDA, "event creation failed");
    }
    d.plan.reset(new Plan());
    g_devs.push_back(std::move(d));
    *out = &g_devs.back();
    return MUON_OK;
}

// ---- tracing ------------------------------------------------------------------

struct Pending {
    cudaEvent_t a, b;
    int kind;
    double flops, bytes;
};

struct Profiler : ProfileSink {
    bool on = false;
    std::vector<Pending> pending;
    std::vector<cudaEvent_t> pool;
    muon_kernel_stats stats[5];
    cudaEvent_t cur = nullptr;
    Profiler() { reset(); }
    void reset() {
        static const char* names[5] = {"momentum_norm", "gemm_tc", "gemm_f32", "scale_apply", "adamw"};
        for (int i = 0; i < 5; ++i) {
            std::memset(&stats[i], 0, sizeof(stats[i]));
            std::strncpy(stats[i].name, names[i], sizeof(stats[i].name) - 1);
        }
    }
    cudaEvent_t get() {
        if (!pool.empty()) {
            cudaEvent_t e = pool.back();
            pool.pop_back();
            return e;
        }
        cudaEvent_t e;
        cudaEventCreate(&e);
        return e;
    }
    void before(cudaStream_t s) override {
        cur = get();
        cudaEventRecord(cur, s);
    }
    void after(cudaStream_t s, int kind, double flops, double bytes) override {
        cudaEvent_t b = get();
        cudaEventRecord(b, s);
        // LaunchRec kinds: MOM, TC, F32, SCALE -> stats slots 0..3
        pending.push_back({cur, b, kind, flops, bytes});
        cur = nullptr;
    }
    void fold() {
        // MUON_PROFILE_VERBOSE=1 prints every traced launch (position in the
        // call, kind, ms, algorithmic TFLOP/s or GB/s) to stderr.
        static const bool verbose = std::getenv("MUON_PROFILE_VERBOSE") != nullptr;
        int pos = 0;
        for (Pending& p : pending) {
            float ms = 0.f;
            cudaEventSynchronize(p.b);
            cudaEventElapsedTime(&ms, p.a, p.b);
            if (verbose)
                std::fprintf(stderr, "muon launch %3d kind %d %9.4f ms %8.2f TFLOP/s %8.1f GB/s\n", pos, p.kind, ms,
                             ms > 0 ? p.flops / (ms * 1e-3) / 1e12 : 0.0, ms > 0 ? p.bytes / (ms * 1e-3) / 1e9 : 0.0);
            ++pos;
            muon_kernel_stats& st = stats[p.kind];
            st.launches += 1;
            st.total_ms += ms;
            st.flops += p.flops;
            st.bytes += p.bytes;
            pool.push_back(p.a);
            pool.push_back(p.b);
        }
        pending.clear();
    }
};
Profiler g_prof;

// True while the bound stream is being captured into a CUDA graph.
bool capturing() {
    cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(g_stream, &st) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return st != cudaStreamCaptureStatusNone;
}

// Order this call's use of the workspace after its last use on another stream.
// Under stream capture the ordering belongs to the capture (it starts after
// the work it was forked from) and to the graph's launches, so no event of
// an earlier, uncaptured call is waited on.
int ws_acquire(DeviceState* ds) {
    if (capturing()) return MUON_OK;
    if (ds->ws_used && ds->ws_stream != g_stream) {
        const cudaError_t e = cudaStreamWaitEvent(g_stream, ds->ws_event, 0);
        if (e != cudaSuccess) return fail(MUON_ERR_CUDA, std::string("stream wait failed: ") + cudaGetErrorString(e));
    }
    return MUON_OK;
}

// Mark the end of this call's use of the workspace on the bound stream (not
// under stream capture: the captured launches run when the graph does).
int ws_release(DeviceState* ds) {
    if (capturing()) return MUON_OK;
    const cudaError_t e = cudaEventRecord(ds->ws_event, g_stream);
    if (e != cudaSuccess) return fail(MUON_ERR_CUDA, std::string("event record failed: ") + cudaGetErrorString(e));
    ds->ws_stream = g_stream;
    ds->ws_used = true;
    return MUON_OK;
}

// An AdamW lane, checked and ready to launch.
struct AdamArgs {
    std::vector<AdamTensor> t;
    AdamLaunch L{};
    double bytes = 0;  // algorithmic HBM bytes
};

// Run rq with `plan` (built for it, or reused when its key matches).  With
// `adam`, the AdamW lane's chunks are appended to the grid of the plan's
// momentum launch.
int run_plan(DeviceState* ds, Plan& plan, const PlanRequest& rq, const AdamArgs* adam) {
    std::string err;
    // a plan is built with allocations, uploads and a stream synchronisation,
    // none of which a stream capture allows: capture only calls whose plan
    // exists (the same call made once before the capture)
    if (capturing() && !plan.same_shape_key(rq))
        return fail(MUON_ERR_UNSUPPORTED,
                    "stream capture needs a built plan: make the same call once before capturing it");
    int wst = ws_acquire(ds);
    if (wst != MUON_OK) return wst;
    if (!plan.same_shape_key(rq)) {
        // tables of the previous plan may still be read by queued kernels
        cudaError_t e = cudaStreamSynchronize(g_stream);
        if (e != cudaSuccess) return fail(MUON_ERR_CUDA, std::string("stream sync failed: ") + cudaGetErrorString(e));
        const int st = plan.build(rq, ds->status, ds->num_sms, g_stream, err);
        if (st != MUON_OK) {
            plan.release();
            return fail(st, err);
        }
    }
    plan.set_scalars(rq.mu, rq.nesterov, rq.lr, rq.clip);
    plan.set_index_base(rq.index_base);
    plan.set_adamw(adam ? &adam->L : nullptr, adam ? adam->bytes : 0.0);
    long long launched = 0;
    const int st = plan.run(g_stream, g_prof.on ? &g_prof : nullptr, &launched, err);
    g_launches += launched;
    wst = ws_release(ds);
    if (st != MUON_OK) return fail(st, err);
    return wst;
}

// ---- argument checks shared by the step entry points (host only) ----------------

// Validate the Muon lane of a step and describe it as a plan request (no device work).
int step_request(void* const* params, const void* const* grads, void* const* momentum, float mu, int nesterov,
                 float lr, const int* shape_list, int count, PlanRequest& rq) {
    if (count < 1) return fail(MUON_ERR_INVALID_ARG, "count must be >= 1");
    if (!params || !grads || !momentum || !shape_list)
        return fail(MUON_ERR_INVALID_ARG, "params, grads, momentum and shape_list must not be NULL");
    if (!std::isfinite(mu) || !std::isfinite(lr)) return fail(MUON_ERR_INVALID_ARG, "mu and lr must be finite");
    for (int i = 0; i < count; ++i) {
        const int r = shape_list[2 * i], c = shape_list[2 * i + 1];
        if (r < 1 || c < 1) return fail(MUON_ERR_INVALID_ARG, "shape_list entries must be >= 1");
        if (!params[i] || !grads[i] || !momentum[i])
            return fail(MUON_ERR_INVALID_ARG, "null pointer in params/grads/momentum");
        rq.rows.push_back(r);
        rq.cols.push_back(c);
        rq.in.push_back(grads[i]);
        rq.mom.push_back(momentum[i]);
        rq.out.push_back(params[i]);
    }
    rq.in_dt = g_cfg.grad_dtype == MUON_DTYPE_F32 ? DT_F32 : DT_BF16;
    rq.mom_dt = g_cfg.momentum_dtype == MUON_DTYPE_F32 ? DT_F32 : DT_BF16;
    rq.out_dt = g_cfg.param_dtype == MUON_DTYPE_F32 ? DT_F32 : DT_BF16;
    rq.is_step = true;
    rq.fp32_path = false;
    rq.form = g_cfg.mode;
    rq.steps = g_cfg.steps;
    rq.coeffs.assign(g_cfg.coeffs, g_cfg.coeffs + 3 * g_cfg.steps);
    rq.restart_mask = g_cfg.restart_mask;
    rq.eps = g_cfg.eps;
    rq.mu = mu;
    rq.nesterov = nesterov ? 1 : 0;
    rq.lr = lr;
    rq.clip = 0.5f * g_cfg.soft_threshold;
    if (!g_shape_scheds.empty()) {
        // each matrix takes the schedule registered for its shape, if any
        std::vector<int> used(g_shape_scheds.size(), -1);
        rq.sched.assign(count, -1);
        for (int i = 0; i < count; ++i) {
            const int n = std::min(rq.rows[i], rq.cols[i]), m = std::max(rq.rows[i], rq.cols[i]);
            for (size_t e = 0; e < g_shape_scheds.size(); ++e) {
                if (g_shape_scheds[e].n != n || g_shape_scheds[e].m != m) continue;
                if (used[e] < 0) {
                    used[e] = static_cast<int>(rq.scheds.size());
                    PlanRequest::Schedule sc;
                    sc.steps = g_shape_scheds[e].steps;
                    sc.coeffs = g_shape_scheds[e].coeffs;
                    rq.scheds.push_back(sc);
                }
                rq.sched[i] = used[e];
                break;
            }
        }
    }
    return MUON_OK;
}

// Validate an AdamW lane and build its launch description (no device work).
int adamw_prepare(void* const* params, const void* const* grads, void* const* exp_avg, void* const* exp_avg_sq,
                  const long long* numels, int count, float lr, float beta1, float beta2, float eps,
                  float weight_decay, int step, AdamArgs& out) {
    if (count < 1) return fail(MUON_ERR_INVALID_ARG, "count must be >= 1");
    if (!params || !grads || !exp_avg || !exp_avg_sq || !numels)
        return fail(MUON_ERR_INVALID_ARG, "params, grads, exp_avg, exp_avg_sq and numels must not be NULL");
    if (step < 1) return fail(MUON_ERR_INVALID_ARG, "step must be >= 1");
    if (!std::isfinite(lr) || !std::isfinite(weight_decay) || !(eps >= 0.f) || !std::isfinite(eps) ||
        !(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f))
        return fail(MUON_ERR_INVALID_ARG, "lr, weight_decay, eps finite; 0 <= beta1, beta2 < 1");
    std::vector<AdamTensor>& t = out.t;
    t.assign(count, AdamTensor{});
    long long chunks = 0;
    const bool pf32 = g_cfg.param_dtype == MUON_DTYPE_F32;
    const bool gf32 = g_cfg.grad_dtype == MUON_DTYPE_F32;
    double elems = 0;
    for (int i = 0; i < count; ++i) {
        if (numels[i] < 1) return fail(MUON_ERR_INVALID_ARG, "numels entries must be >= 1");
        if (!params[i] || !grads[i] || !exp_avg[i] || !exp_avg_sq[i])
            return fail(MUON_ERR_INVALID_ARG, "null pointer in params/grads/exp_avg/exp_avg_sq");
        t[i].p = params[i];
        t[i].g = grads[i];
        t[i].m = static_cast<float*>(exp_avg[i]);
        t[i].v = static_cast<float*>(exp_avg_sq[i]);
        t[i].numel = numels[i];
        t[i].chunk_begin = chunks;
        auto al = [](const void* p, unsigned a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; };
        t[i].vec_ok = numels[i] % 8 == 0 && al(params[i], 16) && al(grads[i], 16) && al(exp_avg[i], 16) &&
                      al(exp_avg_sq[i], 16);
        chunks += (numels[i] + kMomChunk - 1) / kMomChunk;
        elems += static_cast<double>(numels[i]);
    }
    AdamLaunch& L = out.L;
    L.tensors = nullptr;  // set by adamw_upload
    L.ntensors = count;
    L.nchunks = chunks;
    L.p_dt = pf32 ? DT_F32 : DT_BF16;
    L.g_dt = gf32 ? DT_F32 : DT_BF16;
    L.decay = static_cast<float>(1.0 - static_cast<double>(lr) * weight_decay);
    L.beta1 = beta1;
    L.beta2 = beta2;
    L.lr_c1 = static_cast<float>(static_cast<double>(lr) / (1.0 - std::pow(static_cast<double>(beta1), step)));
    L.c2 = static_cast<float>(1.0 / (1.0 - std::pow(static_cast<double>(beta2), step)));
    L.eps = eps;
    out.bytes = elems * ((pf32 ? 8.0 : 4.0) + (gf32 ? 4.0 : 2.0) + 16.0);
    return MUON_OK;
}

// Upload the AdamW tensor table into the library's buffer (after ws_acquire).
int adamw_upload(DeviceState* ds, AdamArgs& aa) {
    // the tensor table lives in a small device buffer owned by the library;
    // a previous launch on the bound stream (or, through ws_acquire, on the
    // stream of the previous call) has read it before this upload runs
    std::vector<AdamTensor>& last = ds->adam_last;
    const std::vector<AdamTensor>& t = aa.t;
    const size_t bytes = sizeof(AdamTensor) * t.size();
    const bool same = last.size() == t.size() && std::memcmp(last.data(), t.data(), bytes) == 0;
    if (!same && capturing())
        return fail(MUON_ERR_UNSUPPORTED,
                    "stream capture needs the AdamW table in place: make the same call once before capturing it");
    if (ds->adam_cap < bytes) {
        if (ds->adam_table) {
            cudaStreamSynchronize(g_stream);
            cudaFree(ds->adam_table);
        }
        ds->adam_table = nullptr;
        ds->adam_cap = 0;
        const char* fault = std::getenv("MUON_FAULT");
        if (fault && !std::strcmp(fault, "alloc"))  // injected failure (see the planner's MUON_FAULT)
            return fail(MUON_ERR_NO_MEMORY, "AdamW table allocation failed (injected: MUON_FAULT=alloc)");
        if (cudaMalloc(&ds->adam_table, bytes) != cudaSuccess) {
            cudaGetLastError();
            return fail(MUON_ERR_NO_MEMORY, "AdamW table allocation failed");
        }
        ds->adam_cap = bytes;
        last.clear();
    }
    if (!same) {
        cudaError_t e = cudaMemcpyAsync(ds->adam_table, t.data(), bytes, cudaMemcpyHostToDevice, g_stream);
        if (e != cudaSuccess) return fail(MUON_ERR_CUDA, std::string("table upload failed: ") + cudaGetErrorString(e));
        last = t;
    }
    aa.L.tensors = static_cast<const AdamTensor*>(ds->adam_table);
    return MUON_OK;
}

int check_device(DeviceState** ds, bool need_tc) {
    const int st = device_state(ds);
    if (st != MUON_OK) return st;
    if (need_tc && (*ds)->cc_major != 10)
        return fail(MUON_ERR_UNSUPPORTED, "the tensor-core path needs an sm_100 GPU (B200)");
    return MUON_OK;
}

// ---- muon_step_offload helpers ---------------------------------------------------

// min(chunks, count) groups of consecutive matrices with about equal weight:
// bounds[0] = 0 < bounds[1] < ... < bounds[g] = count.  Group k closes at the
// first matrix that brings the running total to k/g of the whole, or earlier
// when only one matrix remains for each group still to come.  Returns g.
int offload_groups(const long long* bytes, int count, int chunks, int* bounds) {
    const int g = std::min(chunks, count);
    double total = 0;
    for (int i = 0; i < count; ++i) total += static_cast<double>(bytes[i]);
    const bool flat = !(total > 0);  // all zero: equal counts
    if (flat) total = count;
    bounds[0] = 0;
    int k = 1;
    double acc = 0;
    for (int i = 0; i < count && k < g; ++i) {
        acc += flat ? 1.0 : static_cast<double>(bytes[i]);
        const int remain = count - (i + 1);
        if (remain >= g - k && (acc * g >= total * k || remain == g - k)) bounds[k++] = i + 1;
    }
    bounds[k] = count;
    return k;
}

// True for page-locked (pinned or registered) host memory.
bool pinned_host(const void* p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeHost;
}

// The copy streams, events and plans of ds for `groups` groups (created once).
int offload_resources(DeviceState* ds, int groups) {
    cudaError_t e = cudaSuccess;
    if (!ds->copy_in) e = cudaStreamCreateWithFlags(&ds->copy_in, cudaStreamNonBlocking);
    if (e == cudaSuccess && !ds->copy_out) e = cudaStreamCreateWithFlags(&ds->copy_out, cudaStreamNonBlocking);
    if (e == cudaSuccess && !ds->ev_start) e = cudaEventCreateWithFlags(&ds->ev_start, cudaEventDisableTiming);
    if (e == cudaSuccess && !ds->ev_out) e = cudaEventCreateWithFlags(&ds->ev_out, cudaEventDisableTiming);
    while (e == cudaSuccess && static_cast<int>(ds->ev_in.size()) < groups) {
        cudaEvent_t a = nullptr, b = nullptr;
        e = cudaEventCreateWithFlags(&a, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&b, cudaEventDisableTiming);
        if (e != cudaSuccess) {
            if (a) cudaEventDestroy(a);
            break;
        }
        ds->ev_in.push_back(a);
        ds->ev_done.push_back(b);
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(MUON_ERR_CUDA, std::string("copy stream or event creation failed: ") + cudaGetErrorString(e));
    }
    while (static_cast<int>(ds->chunk_plans.size()) < groups) ds->chunk_plans.emplace_back(new Plan());
    return MUON_OK;
}

}  // namespace

namespace muon {
cudaStream_t bound_stream() { return g_stream; }
void set_last_error(const char* msg) { g_err = msg; }
}  // namespace muon

extern "C" {

int muon_version(void) { return MUON_VERSION; }

int muon_default_config(muon_config* cfg) {
    if (!cfg) return fail(MUON_ERR_INVALID_ARG, "cfg is NULL");
    fill_defaults(cfg);
    return MUON_OK;
}

int muon_set_config(const muon_config* cfg) {
    if (!cfg) return fail(MUON_ERR_INVALID_ARG, "cfg is NULL");
    const int st = check_cfg(*cfg);
    if (st != MUON_OK) return st;
    ensure_cfg();
    g_cfg = *cfg;
    return MUON_OK;
}

int muon_get_config(muon_config* cfg) {
    if (!cfg) return fail(MUON_ERR_INVALID_ARG, "cfg is NULL");
    ensure_cfg();
    *cfg = g_cfg;
    return MUON_OK;
}

int muon_set_stream(void* stream) {
    g_stream = static_cast<cudaStream_t>(stream);
    return MUON_OK;
}

const char* muon_last_error(void) { return g_err.c_str(); }

int muon_release_workspace(void) {
    cudaStreamSynchronize(g_stream);
    int cur = -1;
    cudaGetDevice(&cur);
    for (DeviceState& d : g_devs) {
        if (d.ws_used) {
            cudaSetDevice(d.device);
            cudaEventSynchronize(d.ws_event);  // the last use, on whichever stream
            d.ws_used = false;
        }
        if (d.plan) d.plan->release();
        for (auto& cp : d.chunk_plans) cp->release();
        if (d.adam_table) {
            cudaSetDevice(d.device);
            cudaFree(d.adam_table);
            d.adam_table = nullptr;
            d.adam_cap = 0;
            d.adam_last.clear();
        }
    }
    if (cur >= 0) cudaSetDevice(cur);
    return MUON_OK;
}

int muon_device_status(int* bad_index) {
    if (bad_index) *bad_index = -1;
    DeviceState* ds = nullptr;
    int st = device_state(&ds);
    if (st != MUON_OK) return st;
    cudaError_t e = cudaStreamSynchronize(g_stream);
    if (e != cudaSuccess) return fail(MUON_ERR_CUDA, std::string("stream sync failed: ") + cudaGetErrorString(e));
    DeviceStatus h;
    e = cudaMemcpy(&h, ds->status, sizeof(h), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return fail(MUON_ERR_CUDA, std::string("status read failed: ") + cudaGetErrorString(e));
    const DeviceStatus init{0, 0x7fffffff};
    cudaMemcpy(ds->status, &init, sizeof(init), cudaMemcpyHostToDevice);
    if (bad_index && h.first_bad != 0x7fffffff) *bad_index = h.first_bad;
    if (h.bits & ST_GUARD)
        return fail(MUON_ERR_GUARD, "a workspace guard was overwritten (a write past the end of a workspace region)");
    if (h.bits & ST_TIMEOUT) return fail(MUON_ERR_TIMEOUT, "a kernel's bounded wait ran out");
    if (h.bits & ST_NONFINITE) return fail(MUON_ERR_NONFINITE, "non-finite Frobenius norm");
    return MUON_OK;
}

int muon_orthogonalize(int batch, int m, int n, void* X, const float* coeffs, int steps, int mode) {
    ensure_cfg();
    if (batch < 1 || m < 1 || n < 1) return fail(MUON_ERR_INVALID_ARG, "batch, m and n must be >= 1");
    if (!X) return fail(MUON_ERR_INVALID_ARG, "X is NULL");
    if (steps < 0 || steps > MUON_MAX_STEPS) return fail(MUON_ERR_INVALID_ARG, "steps out of range");
    if (steps > 0 && !coeffs) return fail(MUON_ERR_INVALID_ARG, "coeffs is NULL");
    const int form = mode & MUON_NS_FORM_MASK;
    const bool fp32 = (mode & MUON_PREC_FP32) != 0;
    if ((mode & ~(MUON_NS_FORM_MASK | MUON_PREC_FP32)) != 0 || form > MUON_NS_AUTO)
        return fail(MUON_ERR_INVALID_ARG, "unknown mode bits");
    for (int i = 0; i < 3 * steps; ++i)
        if (!std::isfinite(coeffs[i])) return fail(MUON_ERR_INVALID_ARG, "coeffs must be finite");
    if (static_cast<long long>(m) > (1LL << 30) || static_cast<long long>(n) > (1LL << 30))
        return fail(MUON_ERR_INVALID_ARG, "dimension too large");
    DeviceState* ds = nullptr;
    int st = check_device(&ds, !fp32);
    if (st != MUON_OK) return st;

    PlanRequest rq;
    const int es = fp32 ? 4 : 2;
    for (int b = 0; b < batch; ++b) {
        char* p = static_cast<char*>(X) + static_cast<size_t>(b) * m * n * es;
        rq.rows.push_back(m);
        rq.cols.push_back(n);
        rq.in.push_back(p);
        rq.out.push_back(p);
    }
    rq.in_dt = fp32 ? DT_F32 : DT_BF16;
    rq.out_dt = rq.in_dt;
    rq.is_step = false;
    rq.fp32_path = fp32;
    rq.form = form;
    rq.steps = steps;
    rq.coeffs.assign(coeffs ? coeffs : nullptr, coeffs ? coeffs + 3 * steps : nullptr);
    rq.restart_mask = g_cfg.restart_mask;
    rq.eps = g_cfg.eps;
    rq.device = ds->device;
    return run_plan(ds, *ds->plan, rq, nullptr);
}

int muon_step(void* const* params, const void* const* grads, void* const* momentum, float mu, int nesterov, float lr,
              const int* shape_list, int count) {
    ensure_cfg();
    PlanRequest rq;
    int st = step_request(params, grads, momentum, mu, nesterov, lr, shape_list, count, rq);
    if (st != MUON_OK) return st;
    DeviceState* ds = nullptr;
    st = check_device(&ds, true);
    if (st != MUON_OK) return st;
    rq.device = ds->device;
    return run_plan(ds, *ds->plan, rq, nullptr);
}

int muon_hybrid_step(void* const* params, const void* const* grads, void* const* momentum, float mu, int nesterov,
                     float lr, const int* shape_list, int count, const muon_adamw_lane* adamw) {
    ensure_cfg();
    if (!adamw) return fail(MUON_ERR_INVALID_ARG, "adamw is NULL");
    PlanRequest rq;
    int st = step_request(params, grads, momentum, mu, nesterov, lr, shape_list, count, rq);
    if (st != MUON_OK) return st;
    AdamArgs aa;
    st = adamw_prepare(adamw->params, adamw->grads, adamw->exp_avg, adamw->exp_avg_sq, adamw->numels, adamw->count,
                       adamw->lr, adamw->beta1, adamw->beta2, adamw->eps, adamw->weight_decay, adamw->step, aa);
    if (st != MUON_OK) return st;
    DeviceState* ds = nullptr;
    st = check_device(&ds, true);
    if (st != MUON_OK) return st;
    rq.device = ds->device;
    st = ws_acquire(ds);
    if (st != MUON_OK) return st;
    st = adamw_upload(ds, aa);
    if (st != MUON_OK) return st;
    return run_plan(ds, *ds->plan, rq, &aa);
}

int muon_debug_corrupt_guard(int index) {
    if (index < 0) return fail(MUON_ERR_INVALID_ARG, "index must be >= 0");
    DeviceState* ds = nullptr;
    const int st = device_state(&ds);
    if (st != MUON_OK) return st;
    if (index >= ds->plan->guard_count())
        return fail(MUON_ERR_INVALID_ARG, "no such guard (MUON_DEBUG_CANARY=1 and a plan built by muon_step or "
                                          "muon_orthogonalize are needed)");
    const cudaError_t e = cudaMemsetAsync(ds->plan->guard_addr(index), 0, 1, g_stream);
    if (e != cudaSuccess) return fail(MUON_ERR_CUDA, std::string("memset failed: ") + cudaGetErrorString(e));
    return MUON_OK;
}

int muon_offload_chunks(const long long* bytes, int count, int chunks, int* bounds) {
    if (count < 1 || chunks < 1) return fail(MUON_ERR_INVALID_ARG, "count and chunks must be >= 1");
    if (!bytes || !bounds) return fail(MUON_ERR_INVALID_ARG, "bytes and bounds must not be NULL");
    for (int i = 0; i < count; ++i)
        if (bytes[i] < 0) return fail(MUON_ERR_INVALID_ARG, "bytes must be >= 0");
    return offload_groups(bytes, count, chunks, bounds);
}

int muon_step_offload(void* const* params, const void* const* grads_host, void* const* grads, void* const* momentum,
                      void* const* params_host, float mu, int nesterov, float lr, const int* shape_list, int count,
                      int chunks) {
    ensure_cfg();
    if (chunks < 1) return fail(MUON_ERR_INVALID_ARG, "chunks must be >= 1");
    PlanRequest whole;
    int st = step_request(params, grads, momentum, mu, nesterov, lr, shape_list, count, whole);
    if (st != MUON_OK) return st;
    for (int i = 0; i < count; ++i)
        if ((grads_host && !grads_host[i]) || (params_host && !params_host[i]))
            return fail(MUON_ERR_INVALID_ARG, "null pointer in grads_host/params_host");
    const size_t gsz = g_cfg.grad_dtype == MUON_DTYPE_F32 ? 4 : 2;
    const size_t psz = g_cfg.param_dtype == MUON_DTYPE_F32 ? 4 : 2;
    // groups of about equal copy bytes (both directions)
    std::vector<long long> bytes(count);
    for (int i = 0; i < count; ++i)
        bytes[i] = static_cast<long long>(shape_list[2 * i]) * shape_list[2 * i + 1] *
                   static_cast<long long>((grads_host ? gsz : 0) + (params_host ? psz : 0));
    std::vector<int> bounds(std::min(chunks, count) + 1);
    const int ngroups = offload_groups(bytes.data(), count, chunks, bounds.data());
    std::vector<PlanRequest> rqs(ngroups);
    for (int k = 0; k < ngroups; ++k) {
        const int b = bounds[k], n = bounds[k + 1] - bounds[k];
        st = step_request(params + b, grads + b, momentum + b, mu, nesterov, lr, shape_list + 2 * b, n, rqs[k]);
        if (st != MUON_OK) return st;
        rqs[k].index_base = b;
    }
    DeviceState* ds = nullptr;
    st = check_device(&ds, true);
    if (st != MUON_OK) return st;
    for (int i = 0; i < count; ++i)
        if ((grads_host && !pinned_host(grads_host[i])) || (params_host && !pinned_host(params_host[i])))
            return fail(MUON_ERR_INVALID_ARG, "grads_host/params_host must be page-locked host memory");
    st = offload_resources(ds, ngroups);
    if (st != MUON_OK) return st;
    auto elems = [&](int i) { return static_cast<size_t>(shape_list[2 * i]) * shape_list[2 * i + 1]; };
    auto cuda_fail = [](cudaError_t e, const char* what) {
        return fail(MUON_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
    };
    // the copies start after the work already queued on the bound stream
    cudaError_t e = cudaEventRecord(ds->ev_start, g_stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ds->copy_in, ds->ev_start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ds->copy_out, ds->ev_start, 0);
    if (e != cudaSuccess) return cuda_fail(e, "stream ordering failed");
    // every group's gradients, in order, on the host-to-device stream
    if (grads_host) {
        for (int k = 0; k < ngroups && e == cudaSuccess; ++k) {
            for (int i = bounds[k]; i < bounds[k + 1] && e == cudaSuccess; ++i)
                e = cudaMemcpyAsync(grads[i], grads_host[i], elems(i) * gsz, cudaMemcpyHostToDevice, ds->copy_in);
            if (e == cudaSuccess) e = cudaEventRecord(ds->ev_in[k], ds->copy_in);
        }
    }
    // the groups' steps on the bound stream, each followed by its copy out
    int k = 0;
    for (; k < ngroups && e == cudaSuccess; ++k) {
        if (grads_host) {
            e = cudaStreamWaitEvent(g_stream, ds->ev_in[k], 0);
            if (e != cudaSuccess) break;
        }
        rqs[k].device = ds->device;
        char label[40];
        std::snprintf(label, sizeof(label), "muon offload group %d", k);
        nvtxRangePushA(label);
        st = run_plan(ds, *ds->chunk_plans[k], rqs[k], nullptr);
        nvtxRangePop();
        if (st != MUON_OK) break;
        if (params_host) {
            e = cudaEventRecord(ds->ev_done[k], g_stream);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(ds->copy_out, ds->ev_done[k], 0);
            for (int i = bounds[k]; i < bounds[k + 1] && e == cudaSuccess; ++i)
                e = cudaMemcpyAsync(params_host[i], params[i], elems(i) * psz, cudaMemcpyDeviceToHost, ds->copy_out);
        }
    }
    const std::string run_err = st != MUON_OK ? g_err : std::string();
    // join: work queued on the bound stream after this call follows every copy
    cudaError_t j = cudaEventRecord(ds->ev_out, ds->copy_out);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(g_stream, ds->ev_out, 0);
    if (j == cudaSuccess && grads_host) j = cudaEventRecord(ds->ev_out, ds->copy_in);
    if (j == cudaSuccess && grads_host) j = cudaStreamWaitEvent(g_stream, ds->ev_out, 0);
    if (st != MUON_OK) return fail(st, run_err);
    if (e != cudaSuccess) return cuda_fail(e, "offload copy or ordering failed");
    if (j != cudaSuccess) return cuda_fail(j, "stream join failed");
    return MUON_OK;
}

int muon_set_shape_coeffs(int rows, int cols, const float* coeffs, int steps) {
    if (rows < 1 || cols < 1) return fail(MUON_ERR_INVALID_ARG, "rows and cols must be >= 1");
    if (steps < 0 || steps > MUON_MAX_STEPS) return fail(MUON_ERR_INVALID_ARG, "steps out of range");
    if (steps > 0 && !coeffs) return fail(MUON_ERR_INVALID_ARG, "coeffs is NULL");
    for (int i = 0; i < 3 * steps; ++i)
        if (!std::isfinite(coeffs[i])) return fail(MUON_ERR_INVALID_ARG, "coeffs must be finite");
    const int n = std::min(rows, cols), m = std::max(rows, cols);
    for (ShapeSchedule& e : g_shape_scheds)
        if (e.n == n && e.m == m) {
            e.steps = steps;
            e.coeffs.assign(coeffs, coeffs + 3 * steps);
            return MUON_OK;
        }
    if (static_cast<int>(g_shape_scheds.size()) >= MUON_MAX_SHAPE_SCHEDULES)
        return fail(MUON_ERR_INVALID_ARG, "more than MUON_MAX_SHAPE_SCHEDULES shapes registered");
    ShapeSchedule e;
    e.n = n;
    e.m = m;
    e.steps = steps;
    e.coeffs.assign(coeffs, coeffs + 3 * steps);
    g_shape_scheds.push_back(e);
    return MUON_OK;
}

int muon_get_shape_coeffs(int rows, int cols, float* coeffs, int* steps) {
    if (rows < 1 || cols < 1 || !steps) return fail(MUON_ERR_INVALID_ARG, "rows, cols >= 1 and steps not NULL");
    const int n = std::min(rows, cols), m = std::max(rows, cols);
    for (const ShapeSchedule& e : g_shape_scheds)
        if (e.n == n && e.m == m) {
            *steps = e.steps;
            if (coeffs) std::copy(e.coeffs.begin(), e.coeffs.end(), coeffs);
            return MUON_OK;
        }
    *steps = -1;
    return MUON_OK;
}

int muon_clear_shape_coeffs(void) {
    g_shape_scheds.clear();
    return MUON_OK;
}

int muon_adamw_step(void* const* params, const void* const* grads, void* const* exp_avg, void* const* exp_avg_sq,
                    const long long* numels, int count, float lr, float beta1, float beta2, float eps,
                    float weight_decay, int step) {
    ensure_cfg();
    AdamArgs aa;
    int st = adamw_prepare(params, grads, exp_avg, exp_avg_sq, numels, count, lr, beta1, beta2, eps, weight_decay,
                           step, aa);
    if (st != MUON_OK) return st;
    DeviceState* ds = nullptr;
    st = check_device(&ds, false);
    if (st != MUON_OK) return st;
    st = ws_acquire(ds);
    if (st != MUON_OK) return st;
    st = adamw_upload(ds, aa);
    if (st != MUON_OK) return st;
    if (g_prof.on) g_prof.before(g_stream);
    nvtxRangePushA("muon adamw");
    cudaError_t e = launch_adamw(aa.L, g_stream);
    nvtxRangePop();
    if (e != cudaSuccess) return fail(MUON_ERR_CUDA, std::string("kernel launch failed: ") + cudaGetErrorString(e));
    ++g_launches;
    if (g_prof.on) g_prof.after(g_stream, 4, 0.0, aa.bytes);
    return ws_release(ds);
}

int muon_profile_enable(int on) {
    g_prof.on = on != 0;
    return MUON_OK;
}

int muon_profile_read(muon_kernel_stats* out, int max, int* count) {
    g_prof.fold();
    if (count) *count = 5;
    if (out)
        for (int i = 0; i < max && i < 5; ++i) out[i] = g_prof.stats[i];
    return MUON_OK;
}

int muon_profile_reset(void) {
    g_prof.fold();
    g_prof.reset();
    return MUON_OK;
}

long long muon_launch_count(void) { return g_launches.load(); }

}  // extern "C"
