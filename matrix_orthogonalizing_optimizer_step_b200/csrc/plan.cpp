// Planner: groups matrices by shape, lays out the workspace, writes the
// Newton-Schulz op chain of every group and lowers the chains into grouped
// kernel launches.  See plan.h.
//
// Newton-Schulz forms ([Gram-NS] "ข้อได้เปรียบของอัลกอริทึม" and
// "ความท้าทายด้านความเสถียรและแนวทางแก้ไข"; coefficients from [NanoGPT-Muon]
// "Newton-Schulz 迭代的系数调优"), for X (n x m, n <= m) with X0 = s U,
// s = 1 / (||U||_F + eps):
//
//   standard, per step k:   A = X X^T ;  B = b A + c A^2 ;  X <- a X + B X
//   Gram, per step k:       Z = a I + b R + c R^2 ;  Q <- Z Q ;  R <- Z (Z R)
//                           (R = X X^T at the start of every segment; a restart
//                           before step k sets X <- Q X, R <- X X^T, Q <- I;
//                           the result is Q X)
//
// Precision of the tensor-core path: X, A, B and the bf16 copy of Q used in
// Q X are bf16; the Gram quantities R, Z, Z R, Q are fp16 (the Gram form is
// run in half precision with restarts, as the Gram page describes); every
// product accumulates in fp32 and every stored matrix is rounded once.
#include "plan.h"

#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <tuple>

#include "../../include/muon.h"

namespace muon {
namespace {

enum Buf { X0 = 0, X1, X2, BA, BB, BR, BZ0, BZ1, BZR, BQ0, BQ1, BQBF, NBUF };
constexpr int OUTB = 100;  // the caller's output / parameter, in the caller's layout
enum OpKind { OP_SYRK, OP_PROD, OP_APPLY };
enum SigmaKind { SIG_NONE = 0, SIG_S = 1, SIG_S2 = 2 };

struct OpDesc {
    int kind = OP_PROD;
    int a = -1, b = -1;  // SYRK: a = b = X; PROD: n x n factors; APPLY: a = n x n factor, b = X
    float alpha = 1.f, beta = 0.f, gamma = 0.f, delta = 0.f;
    int sigma = SIG_NONE;
    int c1 = -1, c2 = -1, o1 = -1, o2 = -1;
    bool sym = false;
    bool final = false;
};
using Slot = std::vector<OpDesc>;

struct Group {
    int n = 0, m = 0;
    bool trans = false;
    int form = FORM_STANDARD;
    int steps = 0;              // Newton-Schulz steps of this group's schedule
    std::vector<float> coeffs;  // (a, b, c) of step k at [3k .. 3k+2]
    std::vector<int> mats;
    long long rows_w = 0, cols_w = 0;  // X buffers in the caller's layout
    long long ldx = 0, ldn = 0;
    bool used[NBUF] = {};
    int dt[NBUF] = {};
    size_t off[NBUF] = {};
    long long bstride[NBUF] = {};  // bytes between consecutive matrices
    std::vector<Slot> slots;
};

long long round_up(long long v, long long a) { return (v + a - 1) / a * a; }

// Host-side fault injection for the failure-path tests (MUON_FAULT):
//   alloc    the workspace allocation of a plan build fails (MUON_ERR_NO_MEMORY)
//   launch   the first kernel launch of a call fails (MUON_ERR_CUDA)
//   timeout  the first tile of a chained launch waits on a completion count
//            that is never reached, so its bounded wait runs out
//            (MUON_ERR_TIMEOUT through the device status word)
// No fault is injected on the device: the kernels only see a dependency
// count that no tile will satisfy, and give up after their wait limit.
enum Fault { FAULT_NONE = 0, FAULT_ALLOC, FAULT_LAUNCH, FAULT_TIMEOUT };
int fault_mode() {
    const char* f = std::getenv("MUON_FAULT");
    if (!f) return FAULT_NONE;
    if (!std::strcmp(f, "alloc")) return FAULT_ALLOC;
    if (!std::strcmp(f, "launch")) return FAULT_LAUNCH;
    if (!std::strcmp(f, "timeout")) return FAULT_TIMEOUT;
    return FAULT_NONE;
}

// MUON_TILE_N (read when a plan is built): 256 = persistent launches keep
// 256-wide tiles; 512 = every persistent launch takes 512-wide tiles (tests of
// the wide instance on any shape); unset = chosen per launch.
enum { TILES_AUTO = 0, TILES_NARROW = 1, TILES_WIDE = 2 };
int tile_mode() {
    const char* v = std::getenv("MUON_TILE_N");
    if (v && std::atoi(v) == 256) return TILES_NARROW;
    if (v && std::atoi(v) == 512) return TILES_WIDE;
    return TILES_AUTO;
}

bool canary_mode() {
    const char* v = std::getenv("MUON_DEBUG_CANARY");
    return v && v[0] == '1';
}

// Bound of every device-side wait (MUON_WAIT_LIMIT_MS, 1 ms .. 10 s; default 1 s).
unsigned long long wait_limit_ns() {
    const char* v = std::getenv("MUON_WAIT_LIMIT_MS");
    long long ms = v ? std::atoll(v) : 1000;
    ms = std::max(1LL, std::min(ms, 10000LL));
    return static_cast<unsigned long long>(ms) * 1000000ull;
}

bool restart_at(unsigned mask, int k) { return k > 0 && k < 32 && ((mask >> k) & 1u); }

// ---- op chains ---------------------------------------------------------------

void make_final(OpDesc& op, const PlanRequest& rq) {
    op.final = true;
    op.o1 = OUTB;
    if (rq.is_step) {
        // W <- W - lr * O : the -lr factor is folded into the per-matrix sigma
        op.c2 = OUTB;
        op.gamma = 1.f;
    }
}

void chain_standard(Group& g, const PlanRequest& rq) {
    const int T = g.steps;
    int xcur = X0;
    const int xring[2] = {X1, X2};
    int ring = 0;
    for (int k = 0; k < T; ++k) {
        const float a = g.coeffs[3 * k], b = g.coeffs[3 * k + 1], c = g.coeffs[3 * k + 2];
        OpDesc syrk;
        syrk.kind = OP_SYRK;
        syrk.a = syrk.b = xcur;
        syrk.sym = true;
        syrk.sigma = (k == 0) ? SIG_S2 : SIG_NONE;
        syrk.o1 = BA;
        OpDesc prod;
        prod.kind = OP_PROD;
        prod.a = prod.b = BA;
        prod.sym = true;
        prod.alpha = c;
        prod.beta = b;
        prod.c1 = BA;
        prod.o1 = BB;
        OpDesc app;
        app.kind = OP_APPLY;
        app.a = BB;
        app.b = xcur;
        app.alpha = 1.f;
        app.beta = a;
        app.c1 = xcur;
        app.sigma = (k == 0) ? SIG_S : SIG_NONE;
        if (k == T - 1) {
            make_final(app, rq);
        } else {
            app.o1 = xring[ring];
            ring ^= 1;
            xcur = app.o1;
        }
        g.slots.push_back({syrk});
        g.slots.push_back({prod});
        g.slots.push_back({app});
    }
}

void chain_gram(Group& g, const PlanRequest& rq) {
    const int T = g.steps;
    int xcur = X0;
    bool x_scaled = false;  // X0 still carries the factor s
    const int xring[2] = {X1, X2};
    int ring = 0;
    {
        OpDesc syrk;
        syrk.kind = OP_SYRK;
        syrk.a = syrk.b = xcur;
        syrk.sym = true;
        syrk.sigma = SIG_S2;
        syrk.o1 = BR;
        g.slots.push_back({syrk});
    }
    int qsrc = -1;  // buffer holding Q, -1 = identity (segment start)
    for (int k = 0; k < T; ++k) {
        const float a = g.coeffs[3 * k], b = g.coeffs[3 * k + 1], c = g.coeffs[3 * k + 2];
        if (restart_at(rq.restart_mask, k)) {
            // X <- Q X, R <- X X^T, Q <- I
            OpDesc app;
            app.kind = OP_APPLY;
            app.a = BQBF;
            app.b = xcur;
            app.sigma = x_scaled ? SIG_NONE : SIG_S;
            app.o1 = xring[ring];
            ring ^= 1;
            g.slots.push_back({app});
            xcur = app.o1;
            x_scaled = true;
            OpDesc syrk;
            syrk.kind = OP_SYRK;
            syrk.a = syrk.b = xcur;
            syrk.sym = true;
            syrk.o1 = BR;
            g.slots.push_back({syrk});
            qsrc = -1;
        }
        const bool first = (qsrc == -1);
        const bool last = (k == T - 1) || restart_at(rq.restart_mask, k + 1);
        const int zb = (k & 1) ? BZ1 : BZ0;
        // Z = a I + b R + c R^2
        OpDesc p1;
        p1.kind = OP_PROD;
        p1.a = p1.b = BR;
        p1.sym = true;
        p1.alpha = c;
        p1.beta = b;
        p1.c1 = BR;
        p1.delta = a;
        p1.o1 = (first && last) ? BQBF : zb;  // a one-step segment only needs Q = Z
        g.slots.push_back({p1});
        Slot s2;
        int qnext = zb;  // at a segment start Q = Z (same buffer)
        if (!first) {
            // Q <- Z Q
            OpDesc p4;
            p4.kind = OP_PROD;
            p4.a = zb;
            p4.b = qsrc;
            p4.sym = true;
            p4.o1 = last ? BQBF : (qsrc == BQ0 ? BQ1 : BQ0);
            s2.push_back(p4);
            qnext = p4.o1;
        }
        if (!last) {
            // Z R
            OpDesc p2;
            p2.kind = OP_PROD;
            p2.a = zb;
            p2.b = BR;
            p2.sym = true;
            p2.o1 = BZR;
            s2.push_back(p2);
        }
        if (!s2.empty()) g.slots.push_back(s2);
        if (!last) {
            // R <- Z (Z R)
            OpDesc p3;
            p3.kind = OP_PROD;
            p3.a = zb;
            p3.b = BZR;
            p3.sym = true;
            p3.o1 = BR;
            g.slots.push_back({p3});
        }
        qsrc = qnext;
    }
    OpDesc fin;
    fin.kind = OP_APPLY;
    fin.a = BQBF;
    fin.b = xcur;
    fin.sigma = x_scaled ? SIG_NONE : SIG_S;
    make_final(fin, rq);
    g.slots.push_back({fin});
}

void mark_used(Group& g) {
    for (const Slot& s : g.slots)
        for (const OpDesc& op : s)
            for (int b : {op.a, op.b, op.c1, op.c2, op.o1, op.o2})
                if (b >= 0 && b < NBUF) g.used[b] = true;
    g.used[X0] = true;
}

bool is_x_buf(int b) { return b == X0 || b == X1 || b == X2; }

struct OperandGeom {
    int buf;
    bool mn;
};

void op_geometry(const Group& g, const OpDesc& op, int& M, int& N, int& K, OperandGeom& A, OperandGeom& B) {
    switch (op.kind) {
        case OP_SYRK:
            M = N = g.n;
            K = g.m;
            A = {op.a, g.trans};
            B = {op.b, g.trans};
            break;
        case OP_PROD:
            M = N = K = g.n;
            A = {op.a, false};
            B = {op.b, false};  // symmetric: rows of b are its columns
            break;
        default:  // OP_APPLY
            if (!g.trans) {
                M = g.n, N = g.m, K = g.n;
                A = {op.a, false};
                B = {op.b, true};
            } else {
                M = g.m, N = g.n, K = g.n;
                A = {op.b, false};
                B = {op.a, false};
            }
    }
}

double op_flops(const Group& g, const OpDesc& op) {
    const double n = g.n, m = g.m;
    switch (op.kind) {
        case OP_SYRK: return n * n * m;       // symmetric output: half of 2 n^2 m
        case OP_PROD: return n * n * n;       // symmetric output: half of 2 n^3
        default: return 2.0 * n * n * m;
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder(std::string& err) {
    static EncodeTiledFn fn = nullptr;
    if (fn) return fn;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p) {
        err = "cuTensorMapEncodeTiled unavailable";
        return nullptr;
    }
    fn = reinterpret_cast<EncodeTiledFn>(p);
    return fn;
}

}  // namespace

double ns_flops(int n, int m, int steps, int form, unsigned restart_mask) {
    const double N = n, M = m;
    if (form == FORM_STANDARD) return steps * (3.0 * N * N * M + N * N * N);
    std::vector<int> starts = {0};
    for (int k = 1; k < steps; ++k)
        if (restart_at(restart_mask, k)) starts.push_back(k);
    double total = 0;
    for (size_t i = 0; i < starts.size(); ++i) {
        const int s = starts[i], e = (i + 1 < starts.size()) ? starts[i + 1] : steps;
        total += 3.0 * N * N * M;
        for (int k = s; k < e; ++k) {
            total += N * N * N;
            if (k > s) total += N * N * N;
            if (k < e - 1) total += 2.0 * N * N * N;
        }
    }
    return total;
}

int resolve_form(int n, int m, int steps, int form, unsigned restart_mask) {
    if (form != FORM_AUTO) return form;
    return ns_flops(n, m, steps, FORM_GRAM, restart_mask) < ns_flops(n, m, steps, FORM_STANDARD, restart_mask)
               ? FORM_GRAM
               : FORM_STANDARD;
}

static std::vector<long long> make_key(const PlanRequest& rq) {
    // Everything the tables depend on; mu, nesterov and lr are patched per call.
    std::vector<long long> k;
    k.reserve(16 + rq.rows.size() * 5 + rq.coeffs.size());
    k.push_back(rq.device);
    k.push_back(rq.is_step);
    k.push_back(rq.fp32_path);
    k.push_back(rq.form);
    k.push_back(rq.steps);
    k.push_back(rq.restart_mask);
    int eb;
    std::memcpy(&eb, &rq.eps, sizeof(float));
    k.push_back(eb);
    k.push_back(rq.in_dt);
    k.push_back(rq.mom_dt);
    k.push_back(rq.out_dt);
    auto push_coeffs = [&](const std::vector<float>& cs) {
        for (float c : cs) {
            int bits;
            std::memcpy(&bits, &c, 4);
            k.push_back(bits);
        }
    };
    push_coeffs(rq.coeffs);
    k.push_back(static_cast<long long>(rq.scheds.size()));
    for (const PlanRequest::Schedule& sc : rq.scheds) {
        k.push_back(sc.steps);
        push_coeffs(sc.coeffs);
    }
    for (int si : rq.sched) k.push_back(si);
    k.push_back(fault_mode());
    k.push_back(canary_mode() ? 1 : 0);
    k.push_back(tile_mode());
    k.push_back(static_cast<long long>(wait_limit_ns()));
    for (size_t i = 0; i < rq.rows.size(); ++i) {
        k.push_back(rq.rows[i]);
        k.push_back(rq.cols[i]);
        k.push_back(reinterpret_cast<long long>(rq.in[i]));
        k.push_back(reinterpret_cast<long long>(rq.mom.empty() ? nullptr : rq.mom[i]));
        k.push_back(reinterpret_cast<long long>(rq.out[i]));
    }
    return k;
}

bool Plan::same_shape_key(const PlanRequest& rq) const { return !key_.empty() && make_key(rq) == key_; }

void Plan::set_scalars(float mu, int nesterov, float lr, float clip) {
    for (LaunchRec& l : launches) {
        if (l.kind == LaunchRec::MOM) {
            l.mom.mu = mu;
            l.mom.nesterov = nesterov;
            l.mom.lr = lr;
            l.mom.clip = clip;
        } else if (l.kind == LaunchRec::SCALE) {
            l.sc.lr = lr;
        }
    }
}

void Plan::set_index_base(int base) {
    for (LaunchRec& l : launches)
        if (l.kind == LaunchRec::MOM) l.mom.mat_index_base = base;
}

void Plan::set_adamw(const AdamLaunch* adam, double bytes) {
    for (LaunchRec& l : launches)
        if (l.kind == LaunchRec::MOM) {
            if (adam) {
                l.mom.adam = *adam;
            } else {
                std::memset(&l.mom.adam, 0, sizeof(l.mom.adam));
            }
            l.extra_bytes = adam ? bytes : 0.0;
        }
}

void Plan::release() {
    if (arena_) cudaFree(arena_);
    arena_ = nullptr;
    arena_bytes = 0;
    launches.clear();
    key_.clear();
    guard_offs_.clear();
    d_guard_offs_ = nullptr;
}

int Plan::build(const PlanRequest& rq, DeviceStatus* status, int num_sms, cudaStream_t stream, std::string& err) {
    // ---- key -------------------------------------------------------------------
    launches.clear();
    key_.clear();
    total_flops = 0;
    const int nm = static_cast<int>(rq.rows.size());
    const bool f32 = rq.fp32_path;
    const int tile_m = gemm_tc_tile_m(), tile_n = gemm_tc_tile_n();

    // ---- groups ----------------------------------------------------------------
    std::vector<Group> groups;
    std::map<std::tuple<int, int, int, int, int>, int> gindex;  // (n, m, trans, form, schedule)
    std::vector<int> mat_group(nm), mat_z(nm);
    for (int i = 0; i < nm; ++i) {
        const int r = rq.rows[i], c = rq.cols[i];
        const bool trans = r > c;
        const int n = trans ? c : r, m = trans ? r : c;
        const int si = rq.sched.empty() ? -1 : rq.sched[i];
        const int steps = si < 0 ? rq.steps : rq.scheds[si].steps;
        const int form = steps > 0 ? resolve_form(n, m, steps, rq.form, rq.restart_mask) : FORM_STANDARD;
        auto key = std::make_tuple(n, m, static_cast<int>(trans), form, si);
        auto it = gindex.find(key);
        int gi;
        if (it == gindex.end()) {
            gi = static_cast<int>(groups.size());
            gindex[key] = gi;
            Group g;
            g.n = n;
            g.m = m;
            g.trans = trans;
            g.form = form;
            g.steps = steps;
            g.coeffs = si < 0 ? rq.coeffs : rq.scheds[si].coeffs;
            g.rows_w = r;
            g.cols_w = c;
            g.ldx = round_up(c, 8);
            g.ldn = round_up(n, 8);
            groups.push_back(g);
        } else {
            gi = it->second;
        }
        mat_group[i] = gi;
        mat_z[i] = static_cast<int>(groups[gi].mats.size());
        groups[gi].mats.push_back(i);
    }
    // tile records hold K in 24 bits and batch coordinates in 16 bits
    for (const Group& g : groups) {
        if (!f32 && (static_cast<unsigned>(g.m) > kTileMaxK || g.mats.size() > 65535)) {
            err = "a shape group exceeds the tensor-core tile limits (K < 2^24, at most 65535 matrices of one shape)";
            return MUON_ERR_UNSUPPORTED;
        }
    }
    for (Group& g : groups) {
        if (g.steps > 0) {
            if (g.form == FORM_GRAM)
                chain_gram(g, rq);
            else
                chain_standard(g, rq);
        }
        mark_used(g);
        for (int b = 0; b < NBUF; ++b) {
            if (f32)
                g.dt[b] = DT_F32;
            else if (b == BR || b == BZ0 || b == BZ1 || b == BZR || b == BQ0 || b == BQ1)
                g.dt[b] = DT_F16;
            else
                g.dt[b] = DT_BF16;
        }
    }

    // ---- workspace layout --------------------------------------------------------
    // Regions start 1024-byte aligned.  In the debug canary mode each region
    // is followed, from its exact end, by a guard of kGuardBytes.
    const bool canary = canary_mode();
    guard_offs_.clear();
    size_t cursor = 0;
    auto take = [&](size_t bytes) {
        const size_t o = cursor;
        size_t end = o + bytes;
        if (canary) {
            guard_offs_.push_back(end);
            end += kGuardBytes;
        }
        cursor = static_cast<size_t>(round_up(static_cast<long long>(end), 1024));
        return o;
    };
    for (Group& g : groups) {
        const long long cnt = static_cast<long long>(g.mats.size());
        for (int b = 0; b < NBUF; ++b) {
            if (!g.used[b]) continue;
            const long long rows = is_x_buf(b) ? g.rows_w : g.n;
            const long long ld = is_x_buf(b) ? g.ldx : g.ldn;
            g.bstride[b] = rows * ld * dtype_size(g.dt[b]);
            g.off[b] = take(static_cast<size_t>(g.bstride[b] * cnt));
        }
    }
    // per-matrix chunks of the momentum / normalise kernel
    std::vector<MomMatrix> moms(nm);
    long long nchunks = 0;
    for (int i = 0; i < nm; ++i) {
        const long long numel = static_cast<long long>(rq.rows[i]) * rq.cols[i];
        moms[i].chunk_begin = nchunks;
        moms[i].nchunks = static_cast<int>((numel + kMomChunk - 1) / kMomChunk);
        nchunks += moms[i].nchunks;
    }
    const size_t off_partials = take(sizeof(float) * nchunks);
    const size_t off_counters = take(sizeof(int) * nm);
    const size_t off_scale = take(sizeof(float) * 4 * nm);
    const size_t off_bad = take(sizeof(int) * nm);
    // per-matrix completion counters, then one tile ticket per GEMM launch
    // (at most one per chain slot), all zeroed by the momentum kernel
    const size_t nticket_max = f32 ? 0 : std::max<size_t>(1, [&] {
        size_t n = 0;
        for (const Group& g : groups) n = std::max(n, g.slots.size());
        return n;
    }());
    const size_t off_done = take(sizeof(unsigned) * (nm + nticket_max));
    const size_t off_moms = take(sizeof(MomMatrix) * nm);
    const size_t off_smats = take(sizeof(ScaleMatrix) * nm);

    // ---- count problems / maps ---------------------------------------------------
    size_t nslots = 0;
    for (const Group& g : groups) nslots = std::max(nslots, g.slots.size());
    size_t nprob = 0;
    for (const Group& g : groups)
        for (const Slot& s : g.slots) nprob += s.size() * g.mats.size();
    const size_t off_probs = take((f32 ? sizeof(F32Problem) : sizeof(TcProblem)) * std::max<size_t>(nprob, 1));
    // tiles (upper bound: every tile of every problem)
    size_t ntiles_max = 0;
    if (!f32) {
        for (const Group& g : groups)
            for (const Slot& s : g.slots)
                for (const OpDesc& op : s) {
                    int M, N, K;
                    OperandGeom A, B;
                    op_geometry(g, op, M, N, K, A, B);
                    ntiles_max += static_cast<size_t>((M + tile_m - 1) / tile_m) * ((N + tile_n - 1) / tile_n) *
                                  g.mats.size();
                }
    }
    const size_t off_tiles = take(sizeof(TcTile) * std::max<size_t>(ntiles_max, 1));
    // tensor maps: at most 2 operands per op per group, each with a transposed
    // map when symmetric (deduplicated below)
    size_t nmaps_max = 0;
    for (const Group& g : groups)
        for (const Slot& s : g.slots) nmaps_max += 4 * s.size();
    // TMA store maps: one per workspace buffer of a group, one per caller output
    nmaps_max += groups.size() * NBUF + static_cast<size_t>(nm);
    const size_t off_maps = take(sizeof(CUtensorMap) * std::max<size_t>(nmaps_max, 1));
    // the guard offsets, themselves guarded (their own entry is the last one)
    const size_t off_guards = canary ? take(sizeof(unsigned long long) * (guard_offs_.size() + 1)) : 0;
    const size_t need = cursor;

    // ---- arena -----------------------------------------------------------------
    const int fault = fault_mode();
    if (need > arena_bytes || fault == FAULT_ALLOC) {
        if (arena_) cudaFree(arena_);
        arena_ = nullptr;
        arena_bytes = 0;
        if (fault == FAULT_ALLOC) {
            err = "workspace allocation of " + std::to_string(need) + " bytes failed (injected: MUON_FAULT=alloc)";
            return MUON_ERR_NO_MEMORY;
        }
        if (cudaMalloc(&arena_, need) != cudaSuccess) {
            cudaGetLastError();
            err = "workspace allocation of " + std::to_string(need) + " bytes failed";
            return MUON_ERR_NO_MEMORY;
        }
        arena_bytes = need;
    }
    char* base = static_cast<char*>(arena_);
    status_ = status;
    d_guard_offs_ = canary ? reinterpret_cast<const unsigned long long*>(base + off_guards) : nullptr;
    float* d_partials = reinterpret_cast<float*>(base + off_partials);
    int* d_counters = reinterpret_cast<int*>(base + off_counters);
    float* d_scale = reinterpret_cast<float*>(base + off_scale);
    int* d_bad = reinterpret_cast<int*>(base + off_bad);
    unsigned* d_done = reinterpret_cast<unsigned*>(base + off_done);
    // One chained launch for the whole tensor-core chain (tiles wait on
    // per-matrix completion counters), unless per-slot launches are asked for
    // (per-op tracing) or the co-resident pair count is unknown.
    // Chaining pays where slots are short (few tile rounds per CTA pair, so
    // launch fill and drain dominate); long slots keep one launch per slot.
    // MUON_CHAIN_LAUNCH=1 / MUON_SLOT_LAUNCHES=1 force either mode.
    const int max_pairs = f32 ? 0 : gemm_tc_max_pairs();
    bool chained = false;
    if (!f32 && max_pairs > 0) {
        size_t ntiles_est = 0, nslots_est = 0;
        for (const Group& g : groups) {
            nslots_est = std::max(nslots_est, g.slots.size());
            for (const Slot& sl : g.slots)
                for (const OpDesc& op : sl) {
                    int M, N, K;
                    OperandGeom A, B;
                    op_geometry(g, op, M, N, K, A, B);
                    const size_t tm = (M + tile_m - 1) / tile_m, tn = (N + tile_n - 1) / tile_n;
                    ntiles_est += (op.sym ? (tm * (tm + 1)) / 2 : tm * tn) * g.mats.size();
                }
        }
        const double rounds_per_slot =
            nslots_est ? static_cast<double>(ntiles_est) / nslots_est / max_pairs : 0.0;
        chained = rounds_per_slot < 16.0;
        if (std::getenv("MUON_CHAIN_LAUNCH")) chained = true;
        if (std::getenv("MUON_SLOT_LAUNCHES")) chained = false;
        if (fault == FAULT_TIMEOUT) chained = true;  // the injected wait is a chain dependency
    }
    // Persistent (per-slot) launches of long products use 256 x 512 tiles: a
    // quarter fewer operand bytes per FLOP, but one accumulator (the epilogue
    // no longer overlaps the next tile's main loop), and on symmetric outputs
    // more tile area computed below the diagonal of symmetric outputs (a wide
    // tile whose first half is a lower block skips that half: TILE_LOWER0).
    // A launch takes them when its FLOP-weighted K is at least kWideMinK
    // (shorter, the exposed epilogue costs more than the bytes save) and its
    // wide tiles compute at most kWideMaxArea times the area of its 256-wide
    // ones, K-weighted, and it has at least kWideMinRounds wide tiles per
    // resident CTA pair (with fewer, the epilogues that no longer overlap and
    // the last round's tail dominate).  Chained launches keep 256 x 256 tiles
    // and the double-buffered accumulators.
    constexpr double kWideMinK = 3072.0, kWideMaxArea = 1.08, kWideMinRounds = 4.0;
    const bool wide = !f32 && !chained && tile_mode() != TILES_NARROW;
    // 256-column blocks computed by the 256 x tw tiles of an M x N output
    // (symmetric: tiles wholly below the diagonal are left out, and a wide
    // tile's lower first half is not computed)
    auto block_count = [&](int M, int N, int tw, bool sym) {
        const int per = tw / tile_n;
        long long n = 0;
        for (int bi = 0; bi < (M + tile_m - 1) / tile_m; ++bi)
            for (int bj = 0; bj < (N + tw - 1) / tw; ++bj) {
                if (sym && bi * tile_m > bj * tw + tw - 1) continue;
                n += (sym && per > 1 && bi > bj * per) ? per - 1 : per;
            }
        return n;
    };
    auto tile_count = [&](int M, int N, int tw, bool sym) {
        long long n = 0;
        for (int bi = 0; bi < (M + tile_m - 1) / tile_m; ++bi)
            for (int bj = 0; bj < (N + tw - 1) / tw; ++bj)
                if (!(sym && bi * tile_m > bj * tw + tw - 1)) ++n;
        return n;
    };
    const unsigned long long wait_ns = wait_limit_ns();
    size_t nticket = 0;  // tickets handed out so far (one per GEMM launch)
    auto buf_ptr = [&](const Group& g, int b, int z) -> char* {
        return base + g.off[b] + static_cast<size_t>(g.bstride[b]) * z;
    };

    // ---- momentum / normalise launch -------------------------------------------
    const int u_dt = f32 ? DT_F32 : DT_BF16;
    for (int i = 0; i < nm; ++i) {
        const Group& g = groups[mat_group[i]];
        MomMatrix& mm = moms[i];
        mm.g = rq.in[i];
        mm.m = rq.mom.empty() ? nullptr : rq.mom[i];
        mm.u = buf_ptr(g, X0, mat_z[i]);
        mm.rows = rq.rows[i];
        mm.cols = rq.cols[i];
        mm.ldu = g.ldx;
        auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
        mm.vec_ok = (rq.cols[i] % 8 == 0) && mm.ldu == rq.cols[i] && al(mm.g) && al(mm.u) && (!mm.m || al(mm.m));
    }
    {
        LaunchRec lr;
        lr.kind = LaunchRec::MOM;
        std::snprintf(lr.label, sizeof(lr.label), "muon momentum+norm");
        MomLaunch& L = lr.mom;
        L.mats = reinterpret_cast<const MomMatrix*>(base + off_moms);
        L.nmats = nm;
        L.nchunks = nchunks;
        L.in_dt = rq.in_dt;
        L.mom_dt = rq.mom_dt;
        L.u_dt = u_dt;
        L.has_momentum = rq.is_step ? 1 : 0;
        L.nesterov = rq.nesterov;
        L.mu = rq.mu;
        L.lr = rq.lr;
        L.clip = rq.clip;
        L.eps = rq.eps;
        L.partials = d_partials;
        L.counters = d_counters;
        L.scale = d_scale;
        L.bad = d_bad;
        L.status = status;
        L.mat_index_base = 0;
        L.done = f32 ? nullptr : d_done;
        L.ndone = f32 ? 0 : static_cast<int>(nm + nticket_max);
        double elems = 0;
        for (int i = 0; i < nm; ++i) elems += static_cast<double>(rq.rows[i]) * rq.cols[i];
        const double per = dtype_size(rq.in_dt) + dtype_size(u_dt) + (rq.is_step ? 2.0 * dtype_size(rq.mom_dt) : 0.0);
        lr.bytes = elems * per;
        launches.push_back(lr);
    }

    // ---- steps == 0: elementwise scale / update ---------------------------------
    // matrices whose schedule has no Newton-Schulz step: X0 itself, applied
    // by one elementwise launch
    std::vector<ScaleMatrix> smats;
    bool any_zero_steps = false;
    for (const Group& g : groups) any_zero_steps |= g.steps == 0;
    if (any_zero_steps) {
        long long sc = 0;
        for (int i = 0; i < nm; ++i) {
            const Group& g = groups[mat_group[i]];
            if (g.steps != 0) continue;
            ScaleMatrix s;
            s.u = buf_ptr(g, X0, mat_z[i]);
            s.ldu = g.ldx;
            s.out = rq.out[i];
            s.rows = rq.rows[i];
            s.cols = rq.cols[i];
            s.chunk_begin = sc;
            s.mat = i;
            sc += (s.rows * s.cols + kMomChunk - 1) / kMomChunk;
            smats.push_back(s);
        }
        LaunchRec lr;
        lr.kind = LaunchRec::SCALE;
        std::snprintf(lr.label, sizeof(lr.label), "muon scale");
        ScaleLaunch& L = lr.sc;
        L.mats = reinterpret_cast<const ScaleMatrix*>(base + off_smats);
        L.nmats = static_cast<int>(smats.size());
        L.nchunks = sc;
        L.u_dt = u_dt;
        L.out_dt = rq.out_dt;
        L.update = rq.is_step ? 1 : 0;
        L.lr = rq.lr;
        L.scale = d_scale;
        L.bad = d_bad;
        launches.push_back(lr);
    }

    // ---- GEMM launches -------------------------------------------------------------
    std::vector<TcProblem> tprobs;
    std::vector<F32Problem> fprobs;
    std::vector<TcTile> tiles;
    std::vector<unsigned> mat_tiles_done(nm, 0);  // tiles of each matrix in earlier slots (chained launch)
    // chained launch: matrices ordered by decreasing chain FLOPs (ties: index)
    std::vector<int> mat_rank(nm, 0);
    {
        std::vector<std::pair<double, int>> cost(nm);
        for (int i = 0; i < nm; ++i) {
            const Group& g = groups[mat_group[i]];
            cost[i] = {g.slots.empty() ? 0.0 : ns_flops(g.n, g.m, g.steps, g.form, rq.restart_mask), i};
        }
        std::stable_sort(cost.begin(), cost.end(), [](const std::pair<double, int>& a, const std::pair<double, int>& b) {
            return a.first > b.first;
        });
        for (int r = 0; r < nm; ++r) mat_rank[cost[r].second] = r;
    }
    LaunchRec chain;
    chain.kind = LaunchRec::TC;
    std::snprintf(chain.label, sizeof(chain.label), "muon gemm chain");
    bool chain_open = false;
    std::vector<CUtensorMap> maps;
    std::map<std::tuple<int, int, int>, int> map_index;  // (group, buf, box kind)
    EncodeTiledFn encode = nullptr;
    if (!f32 && nslots > 0) {
        encode = get_encoder(err);
        if (!encode) return MUON_ERR_CUDA;
    }
    enum { BOX_KA = 0, BOX_KB = 1, BOX_MN = 2, BOX_ST = 3 };
    const bool tma_store = !f32 && !(std::getenv("MUON_TMA_STORE") && std::atoi(std::getenv("MUON_TMA_STORE")) == 0);
    auto tmap_dtype = [](int dt) {
        return dt == DT_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                            : (dt == DT_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
    };
    // Store maps: boxes of 64 bytes (32 16-bit or 16 fp32 elements) x 32 rows
    // with the 64-byte swizzle, the epilogue's staging layout.  -1 when the
    // buffer breaks the TMA alignment rules (16-byte base and row pitch).
    auto encode_store_map = [&](void* ptr, int dt, cuuint64_t inner, cuuint64_t outer, cuuint64_t batch,
                                cuuint64_t ld, cuuint64_t bstride) -> int {
        const int es = dtype_size(dt);
        if ((reinterpret_cast<uintptr_t>(ptr) & 15) != 0 || (ld * es) % 16 != 0 || bstride % 16 != 0) return -1;
        if (maps.size() >= 65535 || maps.size() >= nmaps_max) return -1;
        cuuint64_t dims[3] = {inner, outer, batch};
        cuuint64_t strides[2] = {ld * es, bstride};
        cuuint32_t boxd[3] = {static_cast<cuuint32_t>(64 / es), 32, 1};
        cuuint32_t estr[3] = {1, 1, 1};
        CUtensorMap m;
        std::memset(&m, 0, sizeof(m));
        if (encode(&m, tmap_dtype(dt), 3, ptr, dims, strides, boxd, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return -1;
        maps.push_back(m);
        return static_cast<int>(maps.size()) - 1;
    };
    std::map<std::pair<int, int>, int> store_map_index;  // (group, buffer) or (-1 - matrix, OUTB)
    auto get_store_map = [&](int gi, int b, int mi) -> int {
        const auto key = b == OUTB ? std::make_pair(-1 - mi, b) : std::make_pair(gi, b);
        auto it = store_map_index.find(key);
        if (it != store_map_index.end()) return it->second;
        int idx;
        if (b == OUTB) {
            const cuuint64_t r = rq.rows[mi], c = rq.cols[mi];
            idx = encode_store_map(rq.out[mi], rq.out_dt, c, r, 1, c, r * c * dtype_size(rq.out_dt));
        } else {
            const Group& g = groups[gi];
            const bool xb = is_x_buf(b);
            idx = encode_store_map(base + g.off[b], g.dt[b], xb ? g.cols_w : g.n, xb ? g.rows_w : g.n, g.mats.size(),
                                   xb ? g.ldx : g.ldn, g.bstride[b]);
        }
        store_map_index[key] = idx;
        return idx;
    };
    auto get_map = [&](int gi, int b, int box) -> int {
        auto key = std::make_tuple(gi, b, box);
        auto it = map_index.find(key);
        if (it != map_index.end()) return it->second;
        const Group& g = groups[gi];
        const bool xb = is_x_buf(b);
        const cuuint64_t inner = xb ? g.cols_w : g.n;
        const cuuint64_t outer = xb ? g.rows_w : g.n;
        const cuuint64_t ld = xb ? g.ldx : g.ldn;
        const int es = dtype_size(g.dt[b]);
        cuuint64_t dims[3] = {inner, outer, static_cast<cuuint64_t>(g.mats.size())};
        cuuint64_t strides[2] = {ld * es, static_cast<cuuint64_t>(g.bstride[b])};
        // K-major operands: 64 (K) x 128 rows per CTA; MN-major: 64 (MN) x 64 (K)
        cuuint32_t boxd[3] = {64, box == BOX_MN ? 64u : 128u, 1};
        cuuint32_t estr[3] = {1, 1, 1};
        CUtensorMap m;
        std::memset(&m, 0, sizeof(m));
        CUresult r = encode(&m, g.dt[b] == DT_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                            3, base + g.off[b], dims, strides, boxd, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            err = "cuTensorMapEncodeTiled failed (" + std::to_string(static_cast<int>(r)) + ")";
            return -1;
        }
        if (maps.size() >= 65535 || maps.size() >= nmaps_max) {
            err = "too many tensor maps for one plan";
            return -1;
        }
        maps.push_back(m);
        const int idx = static_cast<int>(maps.size()) - 1;
        map_index[key] = idx;
        return idx;
    };

    for (size_t si = 0; si < nslots; ++si) {
        bool slot_wide = false;
        if (wide) {
            double fk = 0.0, fsum = 0.0, area_w = 0.0, area_n = 0.0, tiles_w = 0.0;
            for (const Group& g : groups) {
                if (si >= g.slots.size()) continue;
                for (const OpDesc& op : g.slots[si]) {
                    int M, N, K;
                    OperandGeom A, B;
                    op_geometry(g, op, M, N, K, A, B);
                    const double f = op_flops(g, op) * static_cast<double>(g.mats.size());
                    fk += f * K;
                    fsum += f;
                    const double kw = static_cast<double>(K) * static_cast<double>(g.mats.size());
                    area_n += kw * static_cast<double>(block_count(M, N, tile_n, op.sym));
                    area_w += kw * static_cast<double>(block_count(M, N, gemm_tc_wide_tile_n(), op.sym));
                    tiles_w += static_cast<double>(g.mats.size()) *
                               static_cast<double>(tile_count(M, N, gemm_tc_wide_tile_n(), op.sym));
                }
            }
            slot_wide = tile_mode() == TILES_WIDE ||
                        (fsum > 0.0 && fk >= kWideMinK * fsum && area_w <= kWideMaxArea * area_n &&
                         tiles_w >= kWideMinRounds * std::max(1, max_pairs));
        }
        const int slot_tile_n = slot_wide ? gemm_tc_wide_tile_n() : tile_n;
        LaunchRec lr;
        lr.kind = f32 ? LaunchRec::F32 : LaunchRec::TC;
        std::snprintf(lr.label, sizeof(lr.label), f32 ? "muon gemm_f32 slot %zu" : "muon gemm slot %zu x%d", si,
                      slot_tile_n);
        const size_t prob_begin = f32 ? fprobs.size() : tprobs.size();
        const size_t tile_begin = tiles.size();
        struct TileRef {
            TcTile t;
            int k;
        };
        std::vector<TileRef> ltiles;
        int max_m = 0, max_n = 0;
        for (size_t gi = 0; gi < groups.size(); ++gi) {
            const Group& g = groups[gi];
            if (si >= g.slots.size()) continue;
            for (const OpDesc& op : g.slots[si]) {
                int M, N, K;
                OperandGeom A, B;
                op_geometry(g, op, M, N, K, A, B);
                max_m = std::max(max_m, M);
                max_n = std::max(max_n, N);
                lr.flops += op_flops(g, op) * g.mats.size();
                int amap = -1, bmap = -1, amap_t = -1, bmap_t = -1;
                // n x n operands are symmetric, stored as upper tiles by the
                // tensor-core path: their lower blocks are read transposed
                const bool a_sym = !f32 && !is_x_buf(A.buf), b_sym = !f32 && !is_x_buf(B.buf);
                if (!f32) {
                    amap = get_map(static_cast<int>(gi), A.buf, A.mn ? BOX_MN : BOX_KA);
                    bmap = get_map(static_cast<int>(gi), B.buf, B.mn ? BOX_MN : BOX_KB);
                    if (a_sym) amap_t = get_map(static_cast<int>(gi), A.buf, BOX_MN);
                    if (b_sym) bmap_t = get_map(static_cast<int>(gi), B.buf, BOX_MN);
                    if (amap < 0 || bmap < 0 || (a_sym && amap_t < 0) || (b_sym && bmap_t < 0)) return MUON_ERR_CUDA;
                }
                for (size_t z = 0; z < g.mats.size(); ++z) {
                    const int mi = g.mats[z];
                    Epilogue ep;
                    std::memset(&ep, 0, sizeof(ep));
                    ep.alpha = op.alpha;
                    ep.beta = op.beta;
                    ep.gamma = op.gamma;
                    ep.delta = op.delta;
                    ep.sym = op.sym ? 1 : 0;
                    ep.skip_idx = op.final ? mi : -1;
                    const float* sc = d_scale + 4 * mi;
                    if (op.final && rq.is_step)
                        ep.sigma = sc + (op.sigma == SIG_S ? 2 : 3);  // -lr*s or -lr
                    else
                        ep.sigma = op.sigma == SIG_S ? sc : (op.sigma == SIG_S2 ? sc + 1 : nullptr);
                    auto bind = [&](int b, const void*& p, long long& ld, int& dt) {
                        if (b < 0) {
                            p = nullptr;
                            return;
                        }
                        if (b == OUTB) {
                            p = rq.out[mi];
                            ld = rq.cols[mi];
                            dt = rq.out_dt;
                            return;
                        }
                        p = buf_ptr(g, b, static_cast<int>(z));
                        ld = is_x_buf(b) ? g.ldx : g.ldn;
                        dt = g.dt[b];
                    };
                    const void* tmp = nullptr;
                    bind(op.c1, ep.c1, ep.ldc1, ep.c1_dt);
                    bind(op.c2, ep.c2, ep.ldc2, ep.c2_dt);
                    bind(op.o1, tmp, ep.ldo1, ep.o1_dt);
                    ep.o1 = const_cast<void*>(tmp);
                    tmp = nullptr;
                    bind(op.o2, tmp, ep.ldo2, ep.o2_dt);
                    ep.o2 = const_cast<void*>(tmp);
                    ep.o1_map = -1;
                    ep.o1_z = op.o1 == OUTB ? 0 : static_cast<int>(z);
                    if (tma_store && op.o1 >= 0)
                        ep.o1_map = get_store_map(static_cast<int>(gi), op.o1, mi);
                    if (f32) {
                        F32Problem p;
                        std::memset(&p, 0, sizeof(p));
                        p.M = M;
                        p.N = N;
                        p.K = K;
                        const long long lda = is_x_buf(A.buf) ? g.ldx : g.ldn;
                        const long long ldb = is_x_buf(B.buf) ? g.ldx : g.ldn;
                        p.A = reinterpret_cast<const float*>(buf_ptr(g, A.buf, static_cast<int>(z)));
                        p.a_si = A.mn ? 1 : lda;
                        p.a_sk = A.mn ? lda : 1;
                        p.B = reinterpret_cast<const float*>(buf_ptr(g, B.buf, static_cast<int>(z)));
                        p.b_sk = B.mn ? ldb : 1;
                        p.b_sj = B.mn ? 1 : ldb;
                        p.ep = ep;
                        fprobs.push_back(p);
                    } else {
                        TcProblem p;
                        std::memset(&p, 0, sizeof(p));
                        p.M = M;
                        p.N = N;
                        p.K = K;
                        p.a_map = amap;
                        p.b_map = bmap;
                        p.a_map_t = amap_t;
                        p.b_map_t = bmap_t;
                        p.a_sym = a_sym ? 1 : 0;
                        p.b_sym = b_sym ? 1 : 0;
                        p.a_z = static_cast<int>(z);
                        p.b_z = static_cast<int>(z);
                        p.a_mn = A.mn ? 1 : 0;
                        p.b_mn = B.mn ? 1 : 0;
                        p.fmt = g.dt[A.buf] == DT_F16 ? 0 : 1;
                        p.pad_ = op.sym ? 1 : 0;  // symmetric output: only its upper 256-blocks are stored
                        p.ep = ep;
                        p.ep.sym = 0;  // upper tiles only (tile list below), no mirrored stores
                        const unsigned pi = static_cast<unsigned>(tprobs.size());
                        tprobs.push_back(p);
                        const int tw = slot_tile_n;  // tile width of this launch
                        const int tm = (M + tile_m - 1) / tile_m, tn = (N + tw - 1) / tw;
                        // Tile order within a problem: consecutive tiles (the ones
                        // the pairs work on at once) should share the panels of
                        // the big operand.  A non-transposed apply (n x n factor
                        // times the n x m X) is listed column by column, so the
                        // pairs at work share one or two column panels of X and
                        // the whole small factor; every other product row by row.
                        const bool col_major = op.kind == OP_APPLY && !g.trans;
                        const int outer = col_major ? tn : tm, inner = col_major ? tm : tn;
                        for (int o = 0; o < outer; ++o)
                            for (int i2 = 0; i2 < inner; ++i2) {
                                const int bi = col_major ? i2 : o, bj = col_major ? o : i2;
                                if (op.sym && bi * tile_m > bj * tw + tw - 1) continue;  // wholly below the diagonal
                                TcTile tt;
                                std::memset(&tt, 0, sizeof(tt));
                                tt.problem = pi;
                                tt.kf = static_cast<unsigned>(K) |
                                        static_cast<unsigned>((p.a_mn ? TILE_A_MN : 0) | (p.b_mn ? TILE_B_MN : 0) |
                                                              (p.a_sym ? TILE_A_SYM : 0) | (p.b_sym ? TILE_B_SYM : 0) |
                                                              (p.fmt ? TILE_BF16 : 0))
                                            << 24;
                                tt.a_map = static_cast<unsigned short>(p.a_map);
                                tt.b_map = static_cast<unsigned short>(p.b_map);
                                tt.a_map_t = static_cast<unsigned short>(p.a_sym ? p.a_map_t : 0);
                                tt.b_map_t = static_cast<unsigned short>(p.b_sym ? p.b_map_t : 0);
                                tt.a_z = static_cast<unsigned short>(p.a_z);
                                tt.b_z = static_cast<unsigned short>(p.b_z);
                                tt.bibj = (static_cast<unsigned>(bi) << 16) | static_cast<unsigned>(bj);
                                // wide tile of a symmetric output: a lower first half is skipped
                                if (op.sym && tw > tile_n && bi > bj * (tw / tile_n))
                                    tt.kf |= static_cast<unsigned>(TILE_LOWER0) << 24;
                                tt.mat = static_cast<unsigned>(mi);
                                tt.need = chained ? kTileArrivals * mat_tiles_done[mi] : 0u;
                                ltiles.push_back({tt, K});
                            }
                    }
                }
            }
        }
        if (f32) {
            lr.f32.problems = reinterpret_cast<const F32Problem*>(base + off_probs) + prob_begin;
            lr.f32.nproblems = static_cast<int>(fprobs.size() - prob_begin);
            lr.f32.max_m = max_m;
            lr.f32.max_n = max_n;
            lr.f32.bad = d_bad;
        } else {
            if (chained) {
                // the same matrix order in every slot (largest chain first), so a
                // matrix's earlier-slot tiles are long finished when its next
                // slot's tiles come up
                std::stable_sort(ltiles.begin(), ltiles.end(), [&](const TileRef& x, const TileRef& y) {
                    return mat_rank[x.t.mat] < mat_rank[y.t.mat];
                });
            } else {
                // longest K first: a simple LPT order for the persistent CTAs
                std::stable_sort(ltiles.begin(), ltiles.end(),
                                 [](const TileRef& x, const TileRef& y) { return x.k > y.k; });
            }
            for (const TileRef& t : ltiles) {
                tiles.push_back(t.t);
                ++mat_tiles_done[t.t.mat];
            }
            if (chained) {
                // append this slot to the single chained launch
                chain.flops += lr.flops;
                total_flops += lr.flops;
                chain_open = true;
                continue;
            }
            lr.tc.problems = reinterpret_cast<const TcProblem*>(base + off_probs);
            lr.tc.tiles = reinterpret_cast<const TcTile*>(base + off_tiles) + tile_begin;
            lr.tc.ntiles = static_cast<int>(tiles.size() - tile_begin);
            lr.tc.maps = reinterpret_cast<const CUtensorMap*>(base + off_maps);
            lr.tc.bad = d_bad;
            lr.tc.done = nullptr;
            lr.tc.ticket = d_done + nm + nticket++;
            lr.tc.wait_ns = wait_ns;
            lr.tc.status = status;
            lr.tc.nt = slot_wide ? 2 : 1;
            // CTA pairs: one cluster of 2 per tile, at most one CTA per SM
            lr.grid = 2 * std::max(1, std::min(lr.tc.ntiles, num_sms / 2));
        }
        total_flops += lr.flops;
        launches.push_back(lr);
    }
    if (chain_open) {
        chain.tc.problems = reinterpret_cast<const TcProblem*>(base + off_probs);
        chain.tc.tiles = reinterpret_cast<const TcTile*>(base + off_tiles);
        chain.tc.ntiles = static_cast<int>(tiles.size());
        chain.tc.maps = reinterpret_cast<const CUtensorMap*>(base + off_maps);
        chain.tc.bad = d_bad;
        chain.tc.done = d_done;
        chain.tc.ticket = d_done + nm + nticket++;
        chain.tc.wait_ns = wait_ns;
        chain.tc.status = status;
        chain.tc.nt = 1;
        // one pair per co-resident cluster slot; tiles are claimed in list
        // order, so pairs that are not resident at once delay nothing
        chain.grid = 2 * std::max(1, std::min(chain.tc.ntiles, max_pairs));
        if (fault == FAULT_TIMEOUT && !tiles.empty()) tiles[0].need = 0xFFFFFF00u;  // never reached
        launches.push_back(chain);
    }
    if (nticket > nticket_max) {
        err = "internal: more GEMM launches than tile tickets";
        return MUON_ERR_CUDA;
    }
    fault_launch_ = fault == FAULT_LAUNCH;

    // ---- upload tables -------------------------------------------------------------
    auto up = [&](size_t off, const void* src, size_t bytes) {
        if (bytes == 0) return cudaSuccess;
        return cudaMemcpyAsync(base + off, src, bytes, cudaMemcpyHostToDevice, stream);
    };
    cudaError_t e = cudaSuccess;
    if (e == cudaSuccess) e = up(off_moms, moms.data(), sizeof(MomMatrix) * moms.size());
    if (e == cudaSuccess) e = up(off_smats, smats.data(), sizeof(ScaleMatrix) * smats.size());
    if (e == cudaSuccess && !tprobs.empty()) e = up(off_probs, tprobs.data(), sizeof(TcProblem) * tprobs.size());
    if (e == cudaSuccess && !fprobs.empty()) e = up(off_probs, fprobs.data(), sizeof(F32Problem) * fprobs.size());
    if (e == cudaSuccess && !tiles.empty()) e = up(off_tiles, tiles.data(), sizeof(TcTile) * tiles.size());
    if (e == cudaSuccess && !maps.empty()) e = up(off_maps, maps.data(), sizeof(CUtensorMap) * maps.size());
    if (e == cudaSuccess) e = cudaMemsetAsync(d_counters, 0, sizeof(int) * nm, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(d_done, 0, sizeof(unsigned) * nm, stream);
    if (canary) {
        if (e == cudaSuccess)
            e = up(off_guards, guard_offs_.data(), sizeof(unsigned long long) * guard_offs_.size());
        for (size_t i = 0; i < guard_offs_.size() && e == cudaSuccess; ++i)
            e = cudaMemsetAsync(base + guard_offs_[i], kGuardByte, kGuardBytes, stream);
    }
    if (e != cudaSuccess) {
        err = std::string("table upload failed: ") + cudaGetErrorString(e);
        return MUON_ERR_CUDA;
    }
    key_ = make_key(rq);
    return MUON_OK;
}

int Plan::run(cudaStream_t stream, ProfileSink* prof, long long* launch_counter, std::string& err) {
    if (fault_launch_) {
        err = "kernel launch failed (injected: MUON_FAULT=launch)";
        return MUON_ERR_CUDA;
    }
    for (const LaunchRec& lr : launches) {
        // one NVTX range per launch (host-side enqueue, named by phase and slot)
        nvtxRangePushA(lr.label);
        if (prof) prof->before(stream);
        cudaError_t e = cudaSuccess;
        switch (lr.kind) {
            case LaunchRec::MOM: e = launch_momentum_norm(lr.mom, stream); break;
            case LaunchRec::SCALE: e = launch_scale_apply(lr.sc, stream); break;
            case LaunchRec::TC: e = launch_gemm_tc(lr.tc, lr.grid, stream); break;
            case LaunchRec::F32: e = launch_gemm_f32(lr.f32, stream); break;
        }
        nvtxRangePop();
        if (e != cudaSuccess) {
            err = std::string("kernel launch failed: ") + cudaGetErrorString(e);
            return MUON_ERR_CUDA;
        }
        if (launch_counter) ++*launch_counter;
        if (prof) prof->after(stream, static_cast<int>(lr.kind), lr.flops, lr.bytes + lr.extra_bytes);
    }
    if (d_guard_offs_) {  // debug canary mode: every guard still holds its pattern
        const cudaError_t e = launch_guard_check(arena_, d_guard_offs_, guard_count(), status_, stream);
        if (e != cudaSuccess) {
            err = std::string("guard check launch failed: ") + cudaGetErrorString(e);
            return MUON_ERR_CUDA;
        }
        if (launch_counter) ++*launch_counter;
    }
    return MUON_OK;
}

}  // namespace muon
