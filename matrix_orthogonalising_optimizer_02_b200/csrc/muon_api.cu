// C entry points of the Muon step and of Newton-Schulz orthogonalisation: argument checks,
// workspace layout, and the launch plan
//   momentum + cast + Frobenius partials -> per-matrix scale -> T x (Gram, polynomial,
//   apply) grouped GEMM launches -> scale + weight decay + update,
// following "Muon优化器" (linsight.cn/f25d614e.html): zeropower_via_newtonschulz and
// Muon.step.  Tall matrices (rows > cols) are never transposed: their Gram matrix is
// X^T X (MN-major operands) and the apply step X B, which equals the page's transpose ->
// iterate -> transpose back because B is symmetric.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <functional>
#include <mutex>

#include "runtime.cuh"
#include "simt_async.cuh"

namespace muon {
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// The workspace holds TMA tensor maps (64-byte aligned) and 256-byte aligned buffers.
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

muon_status check_schedule(const muon_ns_schedule* s) {
    if (s == nullptr) return MUON_ERR_INVALID_ARG;
    if (s->n_iters < 0 || s->n_iters > MUON_MAX_NS_ITERS) return MUON_ERR_INVALID_ARG;
    if (s->n_iters > 0 && s->coeffs == nullptr) return MUON_ERR_INVALID_ARG;
    if (s->fp32_mode != 0 && s->fp32_mode != 1) return MUON_ERR_INVALID_ARG;
    if (!s->fp32_mode && (s->n_split_iters < 0 || s->n_split_iters > s->n_iters)) return MUON_ERR_INVALID_ARG;
    if (!(s->eps > 0.f) || !std::isfinite(s->eps)) return MUON_ERR_INVALID_ARG;
    for (int i = 0; i < 3 * s->n_iters; ++i)
        if (!std::isfinite(s->coeffs[i])) return MUON_ERR_INVALID_ARG;
    return MUON_OK;
}

// Shape limits of the bf16 tensor-core path: TMA needs 16-byte row pitches, the tile code
// packs 10-bit block indices.
muon_status check_shape(int rows, int cols, bool fp32) {
    if (rows <= 0 || cols <= 0) return MUON_ERR_INVALID_ARG;
    if (fp32) {
        if (rows > kMaxTileBlocks * kSimtBM || cols > kMaxTileBlocks * kSimtBN) return MUON_ERR_UNSUPPORTED_SHAPE;
        return MUON_OK;
    }
    if (rows % 8 != 0 || cols % 8 != 0) return MUON_ERR_UNSUPPORTED_SHAPE;
    if (rows > kMaxTileBlocks * kTcBM || cols > kMaxTileBlocks * kTcBM) return MUON_ERR_UNSUPPORTED_SHAPE;
    return MUON_OK;
}

long long ew_blocks(long long n) { return (n + kEwElemsPerBlock - 1) / kEwElemsPerBlock; }

// ---------------------------------------------------------------- NS workspace layout
struct NsMat {
    int rows = 0, cols = 0, r = 0, s = 0;
    bool tall = false;
    void* X[2][2] = {{nullptr, nullptr}, {nullptr, nullptr}};  // [ping/pong][hi/lo]
    void* A[2] = {nullptr, nullptr};
    void* B[2] = {nullptr, nullptr};
    float* scale = nullptr;       // device scalar 1 / (||X0|| + eps)
    void* final_out = nullptr;    // optional direct destination of the last apply (bf16)
};

void layout_ns_mat(Arena& ar, NsMat& m, int rows, int cols, bool fp32, bool split) {
    m.rows = rows;
    m.cols = cols;
    m.tall = rows > cols;
    m.r = std::min(rows, cols);
    m.s = std::max(rows, cols);
    const size_t es = fp32 ? 4 : 2;
    const int planes = (!fp32 && split) ? 2 : 1;
    const size_t xb = static_cast<size_t>(rows) * cols * es;
    const size_t ab = static_cast<size_t>(m.r) * m.r * es;
    for (int b = 0; b < 2; ++b)
        for (int p = 0; p < planes; ++p) m.X[b][p] = ar.at(ar.take(xb));
    for (int p = 0; p < planes; ++p) m.A[p] = ar.at(ar.take(ab));
    for (int p = 0; p < planes; ++p) m.B[p] = ar.at(ar.take(ab));
}

size_t ns_mat_bytes(int rows, int cols, bool fp32, bool split) {
    Arena ar;
    NsMat m;
    layout_ns_mat(ar, m, rows, cols, fp32, split);
    return align_up(ar.used, kAlign);
}

int tc_gram_tiles(int r) {
    const int mbs = (r + kTcBM - 1) / kTcBM, nbs = (r + kTcBN - 1) / kTcBN;
    int n = 0;
    for (int mb = 0; mb < mbs; ++mb)
        for (int nb = 0; nb < nbs; ++nb)
            if (kTcBN * nb + kTcBN - 1 >= kTcBM * mb) ++n;
    return n;
}
int tc_apply_tiles(int rows, int cols) {
    return ((rows + kTcBM - 1) / kTcBM) * ((cols + kTcBN - 1) / kTcBN);
}
int simt_tiles(int M, int N) { return ((M + kSimtBM - 1) / kSimtBM) * ((N + kSimtBN - 1) / kSimtBN); }

// Upper bound of the table image of an NS chain over these shapes.
size_t ns_tables_bound(const std::vector<std::pair<int, int>>& shapes, const muon_ns_schedule& sch) {
    size_t b = 0;
    const size_t T = static_cast<size_t>(sch.n_iters);
    for (auto& sh : shapes) {
        const int r = std::min(sh.first, sh.second);
        b += 20 * sizeof(CUtensorMap) + 20 * 128;
        b += 3 * T * (std::max(sizeof(TcProblem), sizeof(SimtProblem)) + 16);
        size_t tiles = sch.fp32_mode ? static_cast<size_t>(2 * simt_tiles(r, r) + simt_tiles(sh.first, sh.second))
                                     : static_cast<size_t>(2 * tc_gram_tiles(r) + tc_apply_tiles(sh.first, sh.second));
        b += T * tiles * sizeof(uint32_t);
    }
    b += 3 * T * 3 * kAlign;
    return b;
}

// TMA boxes: 64 bf16 (128 B) of the contiguous dimension x 128 rows (K-major operand half
// of a pair tile), or 64 x 64 (one MN-major chunk).
constexpr int kBoxK = kTcBM / 2, kBoxMN = 64;

// ---------------------------------------------------------------- NS chain (bf16, tcgen05)
// One stage (0 Gram, 1 polynomial, 2 apply) of iteration t for matrix m: its problem, and its
// tiles (problem index p) appended to `tiles`.  Returns the algorithmic FLOPs.
double ns_stage_problem(TmapPool& pool, NsMat& m, const muon_ns_schedule& sch, int t, int stage, int p,
                        TcProblem& P, std::vector<uint32_t>& tiles, void** final_x) {
    const int T = sch.n_iters;
    const int cur = t & 1, nxt = cur ^ 1;
    const bool split = t < sch.n_split_iters;
    const bool in_lo = t > 0 && (t - 1) < sch.n_split_iters;
    const float a = sch.coeffs[3 * t], b = sch.coeffs[3 * t + 1], c = sch.coeffs[3 * t + 2];
    const bool last = (t == T - 1);
    std::memset(&P, 0, sizeof(P));
    const int r = m.r, s = m.s;
    void* xin0 = m.X[cur][0];
    void* xin1 = in_lo ? m.X[cur][1] : nullptr;
    double flops = 0.0;
    if (stage == 0) {  // A = X X^T (wide) or X^T X (tall)
        const int box_a = m.tall ? kBoxMN : kBoxK, box_b = box_a;
        P.tmA[0] = pool.get(xin0, m.rows, m.cols, box_a);
        P.tmA[1] = pool.get(xin1, m.rows, m.cols, box_a);
        P.tmB[0] = pool.get(xin0, m.rows, m.cols, box_b);
        P.tmB[1] = pool.get(xin1, m.rows, m.cols, box_b);
        P.out[0] = static_cast<__nv_bfloat16*>(m.A[0]);
        P.out[1] = split ? static_cast<__nv_bfloat16*>(m.A[1]) : nullptr;
        P.M = r; P.N = r; P.K = s; P.ld = r;
        P.alpha = 1.f; P.beta = 0.f;
        P.dscale = t == 0 ? m.scale : nullptr;
        P.scale_pow = 2;
        P.flags = kProbSym | (m.tall ? (kProbAMn | kProbBMn) : 0u);
        flops = static_cast<double>(r) * r * s;
    } else if (stage == 1) {  // B = b A + c A A  (A A = A A^T, A symmetric)
        void* a1 = split ? m.A[1] : nullptr;
        P.tmA[0] = pool.get(m.A[0], r, r, kBoxK);
        P.tmA[1] = pool.get(a1, r, r, kBoxK);
        P.tmB[0] = P.tmA[0];
        P.tmB[1] = P.tmA[1];
        P.E[0] = m.A[0];
        P.E[1] = a1;
        P.out[0] = static_cast<__nv_bfloat16*>(m.B[0]);
        P.out[1] = split ? static_cast<__nv_bfloat16*>(m.B[1]) : nullptr;
        P.M = r; P.N = r; P.K = r; P.ld = r;
        P.alpha = c; P.beta = b;
        P.flags = kProbSym;
        flops = static_cast<double>(r) * r * r;
    } else {  // X' = a X + B X (wide) or a X + X B (tall)
        void* b1 = split ? m.B[1] : nullptr;
        if (!m.tall) {
            P.tmA[0] = pool.get(m.B[0], r, r, kBoxK);
            P.tmA[1] = pool.get(b1, r, r, kBoxK);
            P.tmB[0] = pool.get(xin0, m.rows, m.cols, kBoxMN);
            P.tmB[1] = pool.get(xin1, m.rows, m.cols, kBoxMN);
            P.flags = kProbBMn;
        } else {
            P.tmA[0] = pool.get(xin0, m.rows, m.cols, kBoxK);
            P.tmA[1] = pool.get(xin1, m.rows, m.cols, kBoxK);
            P.tmB[0] = pool.get(m.B[0], r, r, kBoxK);
            P.tmB[1] = pool.get(b1, r, r, kBoxK);
            P.flags = 0;
        }
        P.E[0] = xin0;
        P.E[1] = xin1;
        void* out0 = (last && m.final_out) ? m.final_out : m.X[nxt][0];
        P.out[0] = static_cast<__nv_bfloat16*>(out0);
        P.out[1] = split ? static_cast<__nv_bfloat16*>(m.X[nxt][1]) : nullptr;
        P.M = m.rows; P.N = m.cols; P.K = r; P.ld = m.cols;
        P.alpha = 1.f; P.beta = a;
        P.dscale = t == 0 ? m.scale : nullptr;
        P.scale_pow = 1;
        flops = 2.0 * r * r * s;
        if (last) *final_x = out0;
    }
    // split-bf16: hi*hi + hi*lo + lo*hi over the planes present
    tc_set_segments(P, P.tmA[1] ? 2 : 1, P.tmB[1] ? 2 : 1, 1);
    if (stage < 2) {
        const int mbs = (r + kTcBM - 1) / kTcBM, nbs = (r + kTcBN - 1) / kTcBN;
        for (int nb = 0; nb < nbs; ++nb)
            for (int mb = 0; mb < mbs; ++mb)
                if (kTcBN * nb + kTcBN - 1 >= kTcBM * mb) tiles.push_back(tile_code(p, mb, nb));
    } else {
        // Neighbouring CTA pairs (consecutive tiles) share one block of X and sweep the r x r
        // polynomial B, which stays in L2: down the columns for a wide X (B X), along the rows
        // for a tall X (X B).  The other order streams a tall X from DRAM once per column block.
        const int mbs = (m.rows + kTcBM - 1) / kTcBM, nbs = (m.cols + kTcBN - 1) / kTcBN;
        if (!m.tall) {
            for (int nb = 0; nb < nbs; ++nb)
                for (int mb = 0; mb < mbs; ++mb) tiles.push_back(tile_code(p, mb, nb));
        } else {
            for (int mb = 0; mb < mbs; ++mb)
                for (int nb = 0; nb < nbs; ++nb) tiles.push_back(tile_code(p, mb, nb));
        }
    }
    return flops;
}

// Appends the 3T grouped launches of the chain; returns per matrix the buffer holding the
// final X.  (Running the chain in two halves one stage apart, so that each launch paired one
// half's Gram with the other's polynomial or apply, measured 1-3% slower on the GPT-2-small
// set and the low-rank batch.)
muon_status build_ns_tc(Plan& plan, TableImage& img, std::vector<NsMat>& mats, const muon_ns_schedule& sch,
                        unsigned* d_status, std::vector<void*>& final_x) {
    TmapPool pool(img);
    const int T = sch.n_iters;
    const int sms = device_sm_count();
    final_x.assign(mats.size(), nullptr);
    for (size_t i = 0; i < mats.size(); ++i) final_x[i] = mats[i].X[0][0];
    for (int t = 0; t < T; ++t) {
        for (int stage = 0; stage < 3; ++stage) {
            // LPT: problems with the longest K first
            std::vector<int> order(mats.size());
            for (size_t i = 0; i < mats.size(); ++i) order[i] = static_cast<int>(i);
            auto kdim = [&](int i) { return stage == 0 ? mats[i].s : mats[i].r; };
            std::stable_sort(order.begin(), order.end(), [&](int x, int y) { return kdim(x) > kdim(y); });
            std::vector<TcProblem> probs;
            std::vector<uint32_t> tiles;
            double flops = 0.0;
            for (int i : order) {
                TcProblem P;
                flops += ns_stage_problem(pool, mats[i], sch, t, stage, static_cast<int>(probs.size()), P, tiles,
                                          &final_x[i]);
                probs.push_back(P);
            }
            if (pool.failed) return MUON_ERR_CUDA;
            const size_t po = img.add(probs.data(), probs.size() * sizeof(TcProblem), kAlign);
            const size_t to = img.add(tiles.data(), tiles.size() * sizeof(uint32_t), kAlign);
            const TcProblem* dp = img.dev<TcProblem>(po);
            const uint32_t* dt = img.dev<uint32_t>(to);
            const int nt = static_cast<int>(tiles.size());
            plan.steps.push_back({MUON_KERNEL_NS_GEMM, flops, [=](cudaStream_t st) {
                                      return tc_gemm_launch(dp, dt, nt, d_status, sms, st);
                                  }});
        }
    }
    if (pool.failed) return MUON_ERR_CUDA;
    return MUON_OK;
}

// ---------------------------------------------------------------- NS chain (fp32, SIMT)
muon_status build_ns_simt(Plan& plan, TableImage& img, std::vector<NsMat>& mats, const muon_ns_schedule& sch,
                          std::vector<void*>& final_x) {
    const int T = sch.n_iters;
    final_x.assign(mats.size(), nullptr);
    for (size_t i = 0; i < mats.size(); ++i) final_x[i] = mats[i].X[0][0];
    auto vec_ok = [](const void* p, long long ld) { return aligned16(p) && (ld % 4 == 0); };
    for (int t = 0; t < T; ++t) {
        const int cur = t & 1, nxt = cur ^ 1;
        const float a = sch.coeffs[3 * t], b = sch.coeffs[3 * t + 1], c = sch.coeffs[3 * t + 2];
        for (int stage = 0; stage < 3; ++stage) {
            std::vector<SimtProblem> probs;
            std::vector<uint32_t> tiles;
            double flops = 0.0;
            for (size_t i = 0; i < mats.size(); ++i) {
                NsMat& m = mats[i];
                SimtProblem P;
                std::memset(&P, 0, sizeof(P));
                const float* X = static_cast<const float*>(m.X[cur][0]);
                const long long ldx = m.cols, ldr = m.r;
                if (stage == 0) {
                    P.A = X; P.B = X;
                    if (!m.tall) { P.sam = ldx; P.sak = 1; P.sbk = 1; P.sbn = ldx; }
                    else { P.sam = 1; P.sak = ldx; P.sbk = ldx; P.sbn = 1; }
                    P.out = static_cast<float*>(m.A[0]); P.ld_out = ldr;
                    P.M = m.r; P.N = m.r; P.K = m.s;
                    P.alpha = 1.f; P.beta = 0.f;
                    P.dscale = t == 0 ? m.scale : nullptr; P.scale_pow = 2;
                    P.vec_a = P.vec_b = vec_ok(X, ldx);
                } else if (stage == 1) {
                    const float* A = static_cast<const float*>(m.A[0]);
                    P.A = A; P.B = A; P.E = A;
                    P.sam = ldr; P.sak = 1; P.sbk = ldr; P.sbn = 1;
                    P.out = static_cast<float*>(m.B[0]); P.ld_out = ldr; P.ld_e = ldr;
                    P.M = m.r; P.N = m.r; P.K = m.r;
                    P.alpha = c; P.beta = b;
                    P.vec_a = P.vec_b = vec_ok(A, ldr);
                } else {
                    const float* Bm = static_cast<const float*>(m.B[0]);
                    if (!m.tall) { P.A = Bm; P.sam = ldr; P.sak = 1; P.B = X; P.sbk = ldx; P.sbn = 1;
                                   P.vec_a = vec_ok(Bm, ldr); P.vec_b = vec_ok(X, ldx); }
                    else { P.A = X; P.sam = ldx; P.sak = 1; P.B = Bm; P.sbk = ldr; P.sbn = 1;
                           P.vec_a = vec_ok(X, ldx); P.vec_b = vec_ok(Bm, ldr); }
                    P.E = X; P.ld_e = ldx;
                    P.out = static_cast<float*>(m.X[nxt][0]); P.ld_out = ldx;
                    P.M = m.rows; P.N = m.cols; P.K = m.r;
                    P.alpha = 1.f; P.beta = a;
                    P.dscale = t == 0 ? m.scale : nullptr; P.scale_pow = 1;
                    if (t == T - 1) final_x[i] = m.X[nxt][0];
                }
                flops += 2.0 * P.M * P.N * P.K;
                probs.push_back(P);
                const int p = static_cast<int>(probs.size()) - 1;
                const int mbs = (P.M + kSimtBM - 1) / kSimtBM, nbs = (P.N + kSimtBN - 1) / kSimtBN;
                for (int nb = 0; nb < nbs; ++nb)
                    for (int mb = 0; mb < mbs; ++mb) tiles.push_back(tile_code(p, mb, nb));
            }
            const size_t po = img.add(probs.data(), probs.size() * sizeof(SimtProblem), kAlign);
            const size_t to = img.add(tiles.data(), tiles.size() * sizeof(uint32_t), kAlign);
            const SimtProblem* dp = img.dev<SimtProblem>(po);
            const uint32_t* dt = img.dev<uint32_t>(to);
            const int nt = static_cast<int>(tiles.size());
            bool a_kc = false;
            const bool async = simt_async_suits(probs, &a_kc);
            plan.steps.push_back({MUON_KERNEL_SIMT_GEMM, flops, [=](cudaStream_t st) {
                                      return async ? simt_gemm_async_launch(dp, dt, nt, st, a_kc)
                                                   : simt_gemm_launch(dp, dt, nt, st);
                                  }});
        }
    }
    return MUON_OK;
}

SmallParams small_params(const muon_ns_schedule& sch, float beta, int nesterov) {
    SmallParams prm;
    std::memset(&prm, 0, sizeof(prm));
    prm.beta = beta;
    prm.nesterov = nesterov;
    prm.eps = sch.eps;
    prm.n_iters = sch.n_iters;
    for (int i = 0; i < 3 * sch.n_iters; ++i) prm.coeffs[i] = sch.coeffs[i];
    return prm;
}

float scale_for(int rows, int cols, int mode) {
    const double d_out = rows, d_in = cols;
    switch (mode) {
        case MUON_SCALE_MOONLIGHT: return static_cast<float>(0.2 * std::sqrt(std::max(d_out, d_in)));
        case MUON_SCALE_KJ: return static_cast<float>(std::sqrt(std::max(1.0, d_out / d_in)));
        case MUON_SCALE_MUP: return static_cast<float>(std::sqrt(d_out / d_in));
        default: return 1.0f;
    }
}

// ---------------------------------------------------------------- muon_step_batched
struct StepLayout {
    std::vector<std::vector<int>> groups;
    size_t data_bytes = 0;      // largest group
    size_t table_offset = 0;
    size_t table_bound = 0;
};

size_t group_data_bytes(const muon_matrix_desc* d, const std::vector<int>& idx, const muon_ns_schedule& sch) {
    size_t bytes = 0;
    long long blocks = 0;
    for (int i : idx) {
        blocks += ew_blocks(static_cast<long long>(d[i].rows) * d[i].cols);
        bytes += ns_mat_bytes(d[i].rows, d[i].cols, sch.fp32_mode != 0, sch.n_split_iters > 0);
    }
    bytes += align_up(static_cast<size_t>(blocks) * sizeof(double), kAlign);
    bytes += align_up(idx.size() * sizeof(float), kAlign);
    return bytes;
}

size_t step_tables_bound(const muon_matrix_desc* d, int count, const muon_ns_schedule& sch) {
    std::vector<std::pair<int, int>> shapes;
    for (int i = 0; i < count; ++i) shapes.push_back({d[i].rows, d[i].cols});
    size_t b = ns_tables_bound(shapes, sch);
    b += static_cast<size_t>(count) * (sizeof(MomentumItem) + sizeof(UpdateItem) + 2 * sizeof(long long) + 64);
    b += static_cast<size_t>(count) * 8 * kAlign;   // per-group section alignment (<= count groups)
    return align_up(b + 4096, kAlign);
}

muon_status check_step_args(const muon_matrix_desc* descs, int count, const muon_hyper* hp) {
    if (descs == nullptr || hp == nullptr || count <= 0 || count > kMaxTileProblems) return MUON_ERR_INVALID_ARG;
    muon_status st = check_schedule(&hp->ns);
    if (st != MUON_OK) return st;
    if (!std::isfinite(hp->lr) || !std::isfinite(hp->beta) || !std::isfinite(hp->weight_decay))
        return MUON_ERR_INVALID_ARG;
    if (hp->nesterov != 0 && hp->nesterov != 1) return MUON_ERR_INVALID_ARG;
    if (hp->scale_mode < MUON_SCALE_MOONLIGHT || hp->scale_mode > MUON_SCALE_NAIVE) return MUON_ERR_INVALID_ARG;
    for (int i = 0; i < count; ++i) {
        const muon_matrix_desc& d = descs[i];
        if (!d.W || !d.G || !d.M) return MUON_ERR_INVALID_ARG;
        if ((d.w_dtype != MUON_BF16 && d.w_dtype != MUON_F32) || (d.g_dtype != MUON_BF16 && d.g_dtype != MUON_F32))
            return MUON_ERR_INVALID_ARG;
        st = check_shape(d.rows, d.cols, hp->ns.fp32_mode != 0);
        if (st != MUON_OK) return st;
        if (!aligned16(d.W) || !aligned16(d.G) || !aligned16(d.M) || (d.O_out && !aligned16(d.O_out)))
            return MUON_ERR_ALIGNMENT;
    }
    return MUON_OK;
}

// Largest Newton-Schulz data region (X ping-pong, A, B, partial sums) of one group of a step;
// a set needing more runs as consecutive groups that reuse one region.  On the Llama-7B-shaped
// set (40 GB of such data) one group per step took 511 ms, 4 groups 478, 8 groups 460, 16
// groups 463 and 32 groups 468 ms on the same part (groups of about 5 GB are the 8-group
// case), and the step's workspace shrinks from the whole set's data to one group's.
constexpr size_t kStepGroupBytes = static_cast<size_t>(5) << 30;

StepLayout plan_step_layout(const muon_matrix_desc* descs, int count, const muon_hyper* hp, size_t ws_bytes) {
    StepLayout L;
    L.table_bound = step_tables_bound(descs, count, hp->ns);
    const size_t room = ws_bytes > kHeaderBytes + L.table_bound ? ws_bytes - kHeaderBytes - L.table_bound : 0;
    const size_t budget = std::min(room, kStepGroupBytes);
    std::vector<int> cur;
    for (int i = 0; i < count; ++i) {
        std::vector<int> trial = cur;
        trial.push_back(i);
        if (!cur.empty() && group_data_bytes(descs, trial, hp->ns) > budget) {
            L.groups.push_back(cur);
            cur.assign(1, i);
        } else {
            cur.swap(trial);
        }
    }
    if (!cur.empty()) L.groups.push_back(cur);
    for (auto& g : L.groups) L.data_bytes = std::max(L.data_bytes, group_data_bytes(descs, g, hp->ns));
    L.table_offset = kHeaderBytes + align_up(L.data_bytes, kAlign);
    return L;
}

// ---------------------------------------------------------------- host gradients
// Chunks of a host-gradient step: [begin, end) index ranges.  Chunk sizes grow by a factor
// kChunkGrowth (chunk j ends at (g^(j+1) - 1) / (g^target - 1) of the gradient bytes): the
// first chunk, whose copy nothing can hide, is small (2% of the bytes for 8 chunks), and each
// later chunk's copy still finishes within the previous chunk's compute as long as the copy
// runs at least kChunkGrowth times as fast as the step consumes gradients (a B200 over PCIe 5
// copies about 50 GB/s; the bf16 Llama-7B-shaped step consumes about 30 GB/s).
constexpr double kChunkGrowth = 1.5;
std::vector<std::pair<int, int>> host_grad_chunks(const muon_matrix_desc* d, int count) {
    std::vector<size_t> bytes(count);
    size_t total = 0;
    for (int i = 0; i < count; ++i) {
        bytes[i] = static_cast<size_t>(d[i].rows) * d[i].cols * (d[i].g_dtype == MUON_F32 ? 4 : 2);
        total += bytes[i];
    }
    const int target = std::min(count, MUON_HOST_GRAD_CHUNKS);
    std::vector<std::pair<int, int>> chunks;
    size_t acc = 0;
    int begin = 0;
    for (int i = 0; i < count; ++i) {
        acc += bytes[i];
        const double done = (std::pow(kChunkGrowth, static_cast<double>(chunks.size() + 1)) - 1.0) /
                            (std::pow(kChunkGrowth, static_cast<double>(target)) - 1.0);
        const size_t bound = static_cast<size_t>(static_cast<double>(total) * done);
        const int left_items = count - 1 - i, left_chunks = target - static_cast<int>(chunks.size()) - 1;
        const bool may_close = static_cast<int>(chunks.size()) + 1 < target;   // the last chunk takes the rest
        if (i == count - 1 || (may_close && ((acc >= bound && left_items >= left_chunks) || left_items < left_chunks))) {
            chunks.push_back({begin, i + 1});
            begin = i + 1;
        }
    }
    return chunks;
}

size_t grad_slot_bytes(const muon_matrix_desc* d, int begin, int end) {
    size_t b = 0;
    for (int i = begin; i < end; ++i)
        b += align_up(static_cast<size_t>(d[i].rows) * d[i].cols * (d[i].g_dtype == MUON_F32 ? 4 : 2), kAlign);
    return b;
}

// Workspace of a host-gradient step: the call's status header, then two step workspaces and
// two gradient staging slots; chunk c uses step workspace and slot c % 2, so the copy stream
// can fill chunk c + 1's slot and plan tables while chunk c computes.
struct HostGradLayout {
    std::vector<std::pair<int, int>> chunks;
    size_t step_ws = 0;     // one chunk step workspace (largest chunk)
    size_t slot = 0;        // one staging slot
    size_t total = 0;
};

HostGradLayout host_grad_layout(const muon_matrix_desc* d, int count, const muon_hyper* hp) {
    HostGradLayout L;
    L.chunks = host_grad_chunks(d, count);
    for (const auto& c : L.chunks) {
        std::vector<muon_matrix_desc> sub(d + c.first, d + c.second);
        for (auto& x : sub) x.G = x.W;   // placement only: the size depends on shapes and dtypes
        L.step_ws = std::max(L.step_ws, align_up(muon_step_workspace_size(sub.data(), static_cast<int>(sub.size()), hp), kAlign));
        L.slot = std::max(L.slot, grad_slot_bytes(d, c.first, c.second));
    }
    L.total = kHeaderBytes + 2 * L.step_ws + 2 * L.slot;
    return L;
}

__global__ void status_or_kernel(unsigned* dst, const unsigned* src) { atomicOr(dst, *src); }

muon_status step_batched(const muon_matrix_desc* descs, int count, const muon_hyper* hp, void* workspace,
                         size_t ws_bytes, cudaStream_t stream, cudaStream_t upload_stream,
                         const std::function<muon_status()>& before_launch);

cudaStream_t copy_stream_for_device() {
    static std::mutex mu;
    static cudaStream_t streams[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (streams[dev] == nullptr && cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking) != cudaSuccess)
        streams[dev] = nullptr;
    return streams[dev];
}

}  // namespace
}  // namespace muon

using namespace muon;

extern "C" {

const char* muon_status_string(muon_status s) {
    switch (s) {
        case MUON_OK: return "ok";
        case MUON_ERR_INVALID_ARG: return "invalid argument";
        case MUON_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case MUON_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
        case MUON_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case MUON_ERR_CUDA: return "CUDA error";
        case MUON_ERR_NONFINITE: return "non-finite Frobenius norm";
        case MUON_ERR_DEVICE_TIMEOUT: return "a device wait timed out";
        case MUON_ERR_DEVICE_UNDRAINED: return "a device wait timed out and work in flight did not drain";
    }
    return "unknown status";
}

const char* muon_build_info(void) {
    return "muon_b200: sm_100a tcgen05/TMA NS chain, fp32 SIMT GEMM, Woodbury-Cayley; built " __DATE__;
}

size_t muon_step_workspace_size(const muon_matrix_desc* descs, int count, const muon_hyper* hp) {
    if (check_step_args(descs, count, hp) != MUON_OK) return 0;
    const StepLayout L = plan_step_layout(descs, count, hp, SIZE_MAX);
    return L.table_offset + L.table_bound;
}

size_t muon_step_workspace_min(const muon_matrix_desc* descs, int count, const muon_hyper* hp) {
    if (check_step_args(descs, count, hp) != MUON_OK) return 0;
    size_t mx = 0;
    for (int i = 0; i < count; ++i) mx = std::max(mx, group_data_bytes(descs, std::vector<int>{i}, hp->ns));
    return kHeaderBytes + align_up(mx, kAlign) + step_tables_bound(descs, count, hp->ns);
}

muon_status muon_step_batched(const muon_matrix_desc* descs, int count, const muon_hyper* hp, void* workspace,
                              size_t ws_bytes, void* stream_) {
    return step_batched(descs, count, hp, workspace, ws_bytes, static_cast<cudaStream_t>(stream_), nullptr, nullptr);
}

}  // extern "C"

namespace muon {
namespace {
muon_status step_batched(const muon_matrix_desc* descs, int count, const muon_hyper* hp, void* workspace,
                         size_t ws_bytes, cudaStream_t stream, cudaStream_t upload_stream,
                         const std::function<muon_status()>& before_launch) {
    muon_status st = check_step_args(descs, count, hp);
    if (st != MUON_OK) return st;
    if (workspace == nullptr) return MUON_ERR_INVALID_ARG;
    if (!aligned256(workspace)) return MUON_ERR_ALIGNMENT;
    if (ws_bytes < muon_step_workspace_min(descs, count, hp)) return MUON_ERR_WORKSPACE_TOO_SMALL;
    const muon_hyper H = *hp;
    const std::vector<float> coeffs(hp->ns.coeffs, hp->ns.coeffs + 3 * hp->ns.n_iters);
    const std::vector<muon_matrix_desc> D(descs, descs + count);

    KeyWriter kw;
    kw.put(1);  // plan kind: muon step
    kw.put_bytes(D.data(), D.size() * sizeof(muon_matrix_desc));
    kw.put(H.lr); kw.put(H.beta); kw.put(H.weight_decay); kw.put(H.nesterov); kw.put(H.scale_mode);
    kw.put(H.ns.n_iters); kw.put(H.ns.n_split_iters); kw.put(H.ns.fp32_mode); kw.put(H.ns.eps);
    kw.put_bytes(coeffs.data(), coeffs.size() * sizeof(float));
    kw.put(ws_bytes);

    const StepLayout L = plan_step_layout(D.data(), count, &H, ws_bytes);
    if (L.table_offset + L.table_bound > ws_bytes) return MUON_ERR_WORKSPACE_TOO_SMALL;
    unsigned* d_status = static_cast<unsigned*>(workspace);
    uint8_t* ws = static_cast<uint8_t*>(workspace);

    // fp32 mode on small matrices: the whole step of each matrix in one cluster (one launch)
    bool small = H.ns.fp32_mode != 0;
    for (int i = 0; i < count && small; ++i) small = ns_small_fits(D[i].rows, D[i].cols);

    auto build = [&](Plan& plan, TableImage& img) -> muon_status {
        muon_ns_schedule sch = H.ns;
        sch.coeffs = coeffs.data();
        const bool fp32 = sch.fp32_mode != 0;
        if (small) {
            std::vector<SmallItem> items;
            double flops = 0.0;
            for (int i = 0; i < count; ++i) {
                const muon_matrix_desc& d = D[i];
                SmallItem it;
                std::memset(&it, 0, sizeof(it));
                it.G = d.G; it.M = d.M; it.W = d.W; it.O = d.O_out;
                it.rows = d.rows; it.cols = d.cols;
                it.g_f32 = d.g_dtype == MUON_F32; it.w_f32 = d.w_dtype == MUON_F32; it.o_f32 = 1;
                it.decay = 1.0f - H.lr * H.weight_decay;
                it.step = -H.lr * scale_for(d.rows, d.cols, H.scale_mode);
                items.push_back(it);
                const double r = std::min(d.rows, d.cols), sdim = std::max(d.rows, d.cols);
                flops += sch.n_iters * (3.0 * r * r * sdim + r * r * r);
            }
            const SmallItem* di = img.dev<SmallItem>(img.add(items.data(), items.size() * sizeof(SmallItem), kAlign));
            const SmallParams prm = small_params(sch, H.beta, H.nesterov);
            plan.steps.push_back({MUON_KERNEL_SIMT_GEMM, flops, [=](cudaStream_t st) {
                                      return ns_small_launch(di, count, prm, d_status, st);
                                  }});
            if (img.bytes.size() > L.table_bound) return MUON_ERR_WORKSPACE_TOO_SMALL;
            return MUON_OK;
        }
        for (const auto& g : L.groups) {
            Arena ar;
            ar.base = ws + kHeaderBytes;
            long long nblocks = 0;
            for (int i : g) nblocks += ew_blocks(static_cast<long long>(D[i].rows) * D[i].cols);
            double* partials = static_cast<double*>(ar.at(ar.take(static_cast<size_t>(nblocks) * sizeof(double))));
            float* scales = static_cast<float*>(ar.at(ar.take(g.size() * sizeof(float))));
            std::vector<NsMat> mats(g.size());
            std::vector<MomentumItem> mitems;
            std::vector<long long> b0s, nbs;
            long long block0 = 0;
            double mom_bytes = 0.0;
            for (size_t j = 0; j < g.size(); ++j) {
                const muon_matrix_desc& d = D[g[j]];
                layout_ns_mat(ar, mats[j], d.rows, d.cols, fp32, sch.n_split_iters > 0);
                mats[j].scale = scales + j;
                const long long n = static_cast<long long>(d.rows) * d.cols;
                MomentumItem it;
                std::memset(&it, 0, sizeof(it));
                it.G = d.G; it.M = d.M; it.X0 = mats[j].X[0][0]; it.n = n; it.block0 = block0;
                it.g_f32 = d.g_dtype == MUON_F32; it.x_f32 = fp32;
                it.vec = aligned16(it.G) && aligned16(it.M) && aligned16(it.X0);
                mitems.push_back(it);
                b0s.push_back(block0);
                nbs.push_back(ew_blocks(n));
                block0 += ew_blocks(n);
                mom_bytes += n * ((it.g_f32 ? 4.0 : 2.0) + 8.0 + (fp32 ? 4.0 : 2.0));
            }
            const MomentumItem* d_mitems = img.dev<MomentumItem>(img.add(mitems.data(), mitems.size() * sizeof(MomentumItem), kAlign));
            const long long* d_b0 = img.dev<long long>(img.add(b0s.data(), b0s.size() * sizeof(long long), kAlign));
            const long long* d_nb = img.dev<long long>(img.add(nbs.data(), nbs.size() * sizeof(long long), kAlign));
            const int ng = static_cast<int>(g.size());
            const float beta = H.beta, eps = sch.eps;
            const int nesterov = H.nesterov;
            const long long tb = block0;
            plan.steps.push_back({MUON_KERNEL_MOMENTUM, mom_bytes, [=](cudaStream_t s) {
                                      return momentum_cast_launch(d_mitems, ng, tb, beta, nesterov, partials, s);
                                  }});
            plan.steps.push_back({MUON_KERNEL_SCALE, 0.0, [=](cudaStream_t s) {
                                      return frob_scale_launch(d_b0, d_nb, ng, partials, eps, scales, d_status, s);
                                  }});
            std::vector<void*> final_x;
            const muon_status s2 = fp32 ? build_ns_simt(plan, img, mats, sch, final_x)
                                        : build_ns_tc(plan, img, mats, sch, d_status, final_x);
            if (s2 != MUON_OK) return s2;
            std::vector<UpdateItem> uitems;
            double upd_bytes = 0.0;
            for (size_t j = 0; j < g.size(); ++j) {
                const muon_matrix_desc& d = D[g[j]];
                UpdateItem u;
                std::memset(&u, 0, sizeof(u));
                u.W = d.W; u.O = final_x[j]; u.O_out = d.O_out;
                u.dscale = sch.n_iters == 0 ? scales + j : nullptr;
                u.n = static_cast<long long>(d.rows) * d.cols;
                u.block0 = b0s[j];
                u.decay = 1.0f - H.lr * H.weight_decay;
                u.step = -H.lr * scale_for(d.rows, d.cols, H.scale_mode);
                u.w_f32 = d.w_dtype == MUON_F32; u.o_f32 = fp32;
                u.vec = aligned16(u.W) && aligned16(u.O) && (!u.O_out || aligned16(u.O_out));
                uitems.push_back(u);
                upd_bytes += u.n * ((u.w_f32 ? 8.0 : 4.0) + (fp32 ? 4.0 : 2.0) + (d.O_out ? (fp32 ? 4.0 : 2.0) : 0.0));
            }
            const UpdateItem* d_uitems = img.dev<UpdateItem>(img.add(uitems.data(), uitems.size() * sizeof(UpdateItem), kAlign));
            plan.steps.push_back({MUON_KERNEL_UPDATE, upd_bytes, [=](cudaStream_t s) {
                                      return update_launch(d_uitems, ng, tb, s);
                                  }});
        }
        if (img.bytes.size() > L.table_bound) return MUON_ERR_WORKSPACE_TOO_SMALL;
        return MUON_OK;
    };
    return run_plan(kw.k, workspace, L.table_offset, build, stream, upload_stream, before_launch);
}
}  // namespace
}  // namespace muon

extern "C" {

size_t muon_step_host_grad_workspace_size(const muon_matrix_desc* descs, int count, const muon_hyper* hp) {
    if (check_step_args(descs, count, hp) != MUON_OK) return 0;
    return host_grad_layout(descs, count, hp).total;
}

muon_status muon_step_batched_host_grad(const muon_matrix_desc* descs, int count, const muon_hyper* hp,
                                        void* workspace, size_t ws_bytes, void* stream_) {
    muon_status st = check_step_args(descs, count, hp);
    if (st != MUON_OK) return st;
    if (workspace == nullptr) return MUON_ERR_INVALID_ARG;
    if (!aligned256(workspace)) return MUON_ERR_ALIGNMENT;
    for (int i = 0; i < count; ++i) {
        cudaPointerAttributes a;
        if (cudaPointerGetAttributes(&a, descs[i].G) != cudaSuccess || a.type != cudaMemoryTypeHost) {
            cudaGetLastError();
            return MUON_ERR_INVALID_ARG;
        }
    }
    const HostGradLayout L = host_grad_layout(descs, count, hp);
    if (ws_bytes < L.total) return MUON_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    cudaStream_t cs = copy_stream_for_device();
    if (cs == nullptr) return MUON_ERR_CUDA;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    unsigned* status = static_cast<unsigned*>(workspace);
    uint8_t* step_ws[2] = {ws + kHeaderBytes, ws + kHeaderBytes + L.step_ws};
    uint8_t* slots[2] = {ws + kHeaderBytes + 2 * L.step_ws, ws + kHeaderBytes + 2 * L.step_ws + L.slot};

    const int nc = static_cast<int>(L.chunks.size());
    std::vector<cudaEvent_t> ev(static_cast<size_t>(2 * nc + 1), nullptr);
    auto fail = [&](muon_status s) {
        for (cudaEvent_t e : ev)
            if (e) cudaEventDestroy(e);
        return s;
    };
    for (auto& e : ev)
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return fail(MUON_ERR_CUDA);
    // the copy stream joins `stream`'s order (and its capture, if any) here
    if (cudaMemsetAsync(status, 0, sizeof(unsigned), stream) != cudaSuccess ||
        cudaEventRecord(ev[0], stream) != cudaSuccess || cudaStreamWaitEvent(cs, ev[0], 0) != cudaSuccess)
        return fail(MUON_ERR_CUDA);
    for (int c = 0; c < nc; ++c) {
        cudaEvent_t copied = ev[1 + 2 * c], done = ev[2 + 2 * c];
        const int b = L.chunks[c].first, e = L.chunks[c].second;
        // step workspace and slot c % 2 are free once chunk c - 2 has finished on `stream`
        if (c >= 2 && cudaStreamWaitEvent(cs, ev[2 + 2 * (c - 2)], 0) != cudaSuccess) return fail(MUON_ERR_CUDA);
        std::vector<muon_matrix_desc> sub(descs + b, descs + e);
        std::vector<const void*> src(sub.size());
        size_t off = 0;
        for (size_t i = 0; i < sub.size(); ++i) {
            src[i] = sub[i].G;
            sub[i].G = slots[c & 1] + off;
            off += align_up(static_cast<size_t>(sub[i].rows) * sub[i].cols * (sub[i].g_dtype == MUON_F32 ? 4 : 2), kAlign);
        }
        // on the copy stream: the chunk's plan tables (inside step_batched), then its
        // gradients; `stream` waits for both before the chunk's first launch
        auto copy_in = [&]() -> muon_status {
            for (size_t i = 0; i < sub.size(); ++i) {
                const size_t bytes = static_cast<size_t>(sub[i].rows) * sub[i].cols * (sub[i].g_dtype == MUON_F32 ? 4 : 2);
                if (cudaMemcpyAsync(const_cast<void*>(sub[i].G), src[i], bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess)
                    return MUON_ERR_CUDA;
            }
            if (cudaEventRecord(copied, cs) != cudaSuccess || cudaStreamWaitEvent(stream, copied, 0) != cudaSuccess)
                return MUON_ERR_CUDA;
            return MUON_OK;
        };
        st = step_batched(sub.data(), static_cast<int>(sub.size()), hp, step_ws[c & 1], L.step_ws, stream, cs, copy_in);
        if (st != MUON_OK) return fail(st);
        status_or_kernel<<<1, 1, 0, stream>>>(status, reinterpret_cast<const unsigned*>(step_ws[c & 1]));
        if (cudaGetLastError() != cudaSuccess || cudaEventRecord(done, stream) != cudaSuccess)
            return fail(MUON_ERR_CUDA);
    }
    for (cudaEvent_t e : ev) cudaEventDestroy(e);   // released once their work completes
    return MUON_OK;
}

size_t ns_workspace_size(int batch, int rows, int cols, const muon_ns_schedule* sch) {
    if (batch <= 0 || batch > kMaxTileProblems || check_schedule(sch) != MUON_OK ||
        check_shape(rows, cols, sch->fp32_mode != 0) != MUON_OK)
        return 0;
    const long long nb = ew_blocks(static_cast<long long>(rows) * cols) * batch;
    size_t data = align_up(static_cast<size_t>(nb) * sizeof(double), kAlign) +
                  align_up(static_cast<size_t>(batch) * sizeof(float), kAlign) +
                  static_cast<size_t>(batch) * ns_mat_bytes(rows, cols, sch->fp32_mode != 0, sch->n_split_iters > 0);
    std::vector<std::pair<int, int>> shapes(batch, {rows, cols});
    size_t tables = ns_tables_bound(shapes, *sch) +
                    static_cast<size_t>(batch) * (sizeof(MomentumItem) + sizeof(CastItem) + 2 * sizeof(long long)) +
                    8 * kAlign + 4096;
    return kHeaderBytes + align_up(data, kAlign) + align_up(tables, kAlign);
}

muon_status ns_orthogonalize(const void* X_in, int in_dtype, void* X_out, int out_dtype, int batch, int rows,
                             int cols, const muon_ns_schedule* sch_in, void* workspace, size_t ws_bytes,
                             void* stream_) {
    if (X_in == nullptr || X_out == nullptr || workspace == nullptr) return MUON_ERR_INVALID_ARG;
    if ((in_dtype != MUON_BF16 && in_dtype != MUON_F32) || (out_dtype != MUON_BF16 && out_dtype != MUON_F32))
        return MUON_ERR_INVALID_ARG;
    if (batch <= 0 || batch > kMaxTileProblems) return MUON_ERR_INVALID_ARG;
    muon_status st = check_schedule(sch_in);
    if (st != MUON_OK) return st;
    st = check_shape(rows, cols, sch_in->fp32_mode != 0);
    if (st != MUON_OK) return st;
    if (!aligned16(X_in) || !aligned16(X_out) || !aligned256(workspace)) return MUON_ERR_ALIGNMENT;
    const size_t need = ns_workspace_size(batch, rows, cols, sch_in);
    if (ws_bytes < need) return MUON_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    const muon_ns_schedule S = *sch_in;
    const std::vector<float> coeffs(S.coeffs, S.coeffs + 3 * S.n_iters);

    KeyWriter kw;
    kw.put(2);  // plan kind: ns_orthogonalize
    kw.put(X_in); kw.put(in_dtype); kw.put(X_out); kw.put(out_dtype);
    kw.put(batch); kw.put(rows); kw.put(cols);
    kw.put(S.n_iters); kw.put(S.n_split_iters); kw.put(S.fp32_mode); kw.put(S.eps);
    kw.put_bytes(coeffs.data(), coeffs.size() * sizeof(float));
    kw.put(ws_bytes);

    const bool fp32 = S.fp32_mode != 0;
    const long long n = static_cast<long long>(rows) * cols;
    const long long nb1 = ew_blocks(n);
    const size_t data = align_up(static_cast<size_t>(nb1 * batch) * sizeof(double), kAlign) +
                        align_up(static_cast<size_t>(batch) * sizeof(float), kAlign) +
                        static_cast<size_t>(batch) * ns_mat_bytes(rows, cols, fp32, S.n_split_iters > 0);
    const size_t table_offset = kHeaderBytes + align_up(data, kAlign);
    unsigned* d_status = static_cast<unsigned*>(workspace);
    uint8_t* ws = static_cast<uint8_t*>(workspace);

    const bool small = fp32 && ns_small_fits(rows, cols);
    auto build = [&](Plan& plan, TableImage& img) -> muon_status {
        muon_ns_schedule sch = S;
        sch.coeffs = coeffs.data();
        if (small) {   // fp32 mode on small matrices: one cluster per matrix, one launch
            std::vector<SmallItem> items;
            const size_t in_es = in_dtype == MUON_F32 ? 4 : 2, out_es = out_dtype == MUON_F32 ? 4 : 2;
            for (int i = 0; i < batch; ++i) {
                SmallItem it;
                std::memset(&it, 0, sizeof(it));
                it.G = static_cast<const uint8_t*>(X_in) + static_cast<size_t>(i) * n * in_es;
                it.O = static_cast<uint8_t*>(X_out) + static_cast<size_t>(i) * n * out_es;
                it.rows = rows; it.cols = cols;
                it.g_f32 = in_dtype == MUON_F32; it.o_f32 = out_dtype == MUON_F32;
                items.push_back(it);
            }
            const SmallItem* di = img.dev<SmallItem>(img.add(items.data(), items.size() * sizeof(SmallItem), kAlign));
            const SmallParams prm = small_params(sch, 0.f, 0);
            const double r = std::min(rows, cols), sdim = std::max(rows, cols);
            const double flops = static_cast<double>(batch) * sch.n_iters * (3.0 * r * r * sdim + r * r * r);
            plan.steps.push_back({MUON_KERNEL_SIMT_GEMM, flops, [=](cudaStream_t st) {
                                      return ns_small_launch(di, batch, prm, d_status, st);
                                  }});
            if (table_offset + img.bytes.size() > ws_bytes) return MUON_ERR_WORKSPACE_TOO_SMALL;
            return MUON_OK;
        }
        Arena ar;
        ar.base = ws + kHeaderBytes;
        double* partials = static_cast<double*>(ar.at(ar.take(static_cast<size_t>(nb1 * batch) * sizeof(double))));
        float* scales = static_cast<float*>(ar.at(ar.take(static_cast<size_t>(batch) * sizeof(float))));
        std::vector<NsMat> mats(batch);
        std::vector<MomentumItem> items;
        std::vector<long long> b0s, nbs;
        const size_t in_es = in_dtype == MUON_F32 ? 4 : 2, out_es = out_dtype == MUON_F32 ? 4 : 2;
        const bool direct = !fp32 && out_dtype == MUON_BF16 && S.n_iters > 0;
        for (int i = 0; i < batch; ++i) {
            layout_ns_mat(ar, mats[i], rows, cols, fp32, S.n_split_iters > 0);
            mats[i].scale = scales + i;
            if (direct) mats[i].final_out = static_cast<uint8_t*>(X_out) + static_cast<size_t>(i) * n * out_es;
            MomentumItem it;
            std::memset(&it, 0, sizeof(it));
            it.G = static_cast<const uint8_t*>(X_in) + static_cast<size_t>(i) * n * in_es;
            it.M = nullptr;
            it.X0 = mats[i].X[0][0];
            it.n = n;
            it.block0 = nb1 * i;
            it.g_f32 = in_dtype == MUON_F32;
            it.x_f32 = fp32;
            it.vec = aligned16(it.G) && aligned16(it.X0);
            items.push_back(it);
            b0s.push_back(nb1 * i);
            nbs.push_back(nb1);
        }
        const MomentumItem* d_items = img.dev<MomentumItem>(img.add(items.data(), items.size() * sizeof(MomentumItem), kAlign));
        const long long* d_b0 = img.dev<long long>(img.add(b0s.data(), b0s.size() * sizeof(long long), kAlign));
        const long long* d_nb = img.dev<long long>(img.add(nbs.data(), nbs.size() * sizeof(long long), kAlign));
        const long long tb = nb1 * batch;
        const float eps = sch.eps;
        const double cast_bytes = static_cast<double>(n) * batch * (in_es + (fp32 ? 4 : 2));
        plan.steps.push_back({MUON_KERNEL_MOMENTUM, cast_bytes, [=](cudaStream_t s) {
                                  return momentum_cast_launch(d_items, batch, tb, 0.f, 0, partials, s);
                              }});
        plan.steps.push_back({MUON_KERNEL_SCALE, 0.0, [=](cudaStream_t s) {
                                  return frob_scale_launch(d_b0, d_nb, batch, partials, eps, scales, d_status, s);
                              }});
        std::vector<void*> final_x;
        const muon_status s2 = fp32 ? build_ns_simt(plan, img, mats, sch, final_x)
                                    : build_ns_tc(plan, img, mats, sch, d_status, final_x);
        if (s2 != MUON_OK) return s2;
        if (!direct) {
            std::vector<CastItem> citems;
            for (int i = 0; i < batch; ++i) {
                CastItem c;
                std::memset(&c, 0, sizeof(c));
                c.src = final_x[i];
                c.dst = static_cast<uint8_t*>(X_out) + static_cast<size_t>(i) * n * out_es;
                c.dscale = S.n_iters == 0 ? scales + i : nullptr;
                c.n = n;
                c.block0 = nb1 * i;
                c.src_f32 = fp32;
                c.dst_f32 = out_dtype == MUON_F32;
                c.vec = aligned16(c.src) && aligned16(c.dst);
                citems.push_back(c);
            }
            const CastItem* d_c = img.dev<CastItem>(img.add(citems.data(), citems.size() * sizeof(CastItem), kAlign));
            const double bytes = static_cast<double>(n) * batch * ((fp32 ? 4 : 2) + out_es);
            plan.steps.push_back({MUON_KERNEL_MISC, bytes, [=](cudaStream_t s) {
                                      return cast_launch(d_c, batch, tb, s);
                                  }});
        }
        if (table_offset + img.bytes.size() > ws_bytes) return MUON_ERR_WORKSPACE_TOO_SMALL;
        return MUON_OK;
    };
    return run_plan(kw.k, workspace, table_offset, build, stream);
}

muon_status muon_workspace_device_status(void* workspace, size_t ws_bytes, int* status_out, void* stream_) {
    if (workspace == nullptr || status_out == nullptr || ws_bytes < kHeaderBytes) return MUON_ERR_INVALID_ARG;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    unsigned word = 0;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MUON_ERR_CUDA;
    if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return MUON_ERR_CUDA;
    if (cudaMemset(workspace, 0, sizeof(word)) != cudaSuccess) return MUON_ERR_CUDA;
    *status_out = (word & kDevErrUndrained)   ? MUON_ERR_DEVICE_UNDRAINED
                  : (word & kDevErrTimeout)   ? MUON_ERR_DEVICE_TIMEOUT
                  : (word & kDevErrNonfinite) ? MUON_ERR_NONFINITE
                                              : MUON_OK;
    return MUON_OK;
}

}  // extern "C"
