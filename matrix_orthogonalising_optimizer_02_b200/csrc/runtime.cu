// Host runtime: plan cache with pinned table images, per-kind device timing, tensor maps.
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cstdio>
#include <mutex>

#include "runtime.cuh"

namespace muon {

namespace {

std::mutex g_mu;
std::vector<std::unique_ptr<Plan>> g_plans;   // most recently used last
constexpr size_t kMaxPlans = 32;

struct TimingRec {
    int kind;
    double work;
    cudaEvent_t e0, e1;
};
struct Timing {
    bool enabled = false;
    std::vector<TimingRec> pending;
    double ms[MUON_KERNEL_KINDS] = {};
    long long launches[MUON_KERNEL_KINDS] = {};
    double work[MUON_KERNEL_KINDS] = {};
} g_timing;

void drain_timing_locked() {
    for (auto& r : g_timing.pending) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.e1) == cudaSuccess && cudaEventElapsedTime(&ms, r.e0, r.e1) == cudaSuccess) {
            g_timing.ms[r.kind] += ms;
            g_timing.launches[r.kind] += 1;
            g_timing.work[r.kind] += r.work;
        }
        cudaEventDestroy(r.e0);
        cudaEventDestroy(r.e1);
    }
    g_timing.pending.clear();
}

}  // namespace

Plan::~Plan() {
    if (last_use) {
        if (recorded) cudaEventSynchronize(last_use);   // the last table copy has finished
        cudaEventDestroy(last_use);
    }
    if (pinned) cudaFreeHost(pinned);
    cudaGetLastError();   // leave no error of this cleanup pending for the caller's next check
}

namespace {
thread_local char g_last_error[256] = "";
}

muon_status cuda_error(cudaError_t e, const char* where) {
    std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
    return MUON_ERR_CUDA;
}

muon_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MUON_OK : cuda_error(e, "CUDA call"); }

int device_sm_count() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
    return sms;
}

muon_status run_plan(const std::vector<uint8_t>& key_in, void* workspace, size_t table_offset,
                     const std::function<muon_status(Plan&, TableImage&)>& build, cudaStream_t stream,
                     cudaStream_t upload_stream, const std::function<muon_status()>& before_launch) {
    std::lock_guard<std::mutex> lk(g_mu);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
    // An error left pending by earlier, unrelated work would otherwise be reported by the
    // first launch check below as this call's own failure: clear it, and name it if this call
    // then fails.
    const cudaError_t pending = cudaGetLastError();
    KeyWriter kw;
    kw.put_bytes(key_in.data(), key_in.size());
    kw.put(dev);
    kw.put(workspace);
    kw.put(table_offset);

    Plan* plan = nullptr;
    for (size_t i = 0; i < g_plans.size(); ++i) {
        if (g_plans[i]->key == kw.k) {
            std::unique_ptr<Plan> p = std::move(g_plans[i]);
            g_plans.erase(g_plans.begin() + static_cast<long>(i));
            g_plans.push_back(std::move(p));
            plan = g_plans.back().get();
            break;
        }
    }
    if (plan == nullptr) {
        auto p = std::make_unique<Plan>();
        p->key = kw.k;
        TableImage img;
        img.dev_base = static_cast<uint8_t*>(workspace) + table_offset;
        const muon_status st = build(*p, img);
        if (st != MUON_OK) return st;
        p->table_bytes = img.bytes.size();
        p->dev_tables = img.dev_base;
        if (p->table_bytes) {
            e = cudaHostAlloc(reinterpret_cast<void**>(&p->pinned), p->table_bytes, cudaHostAllocDefault);
            if (e != cudaSuccess) return cuda_error(e, "cudaHostAlloc of the plan tables");
            std::memcpy(p->pinned, img.bytes.data(), p->table_bytes);
        }
        e = cudaEventCreateWithFlags(&p->last_use, cudaEventDisableTiming);
        if (e != cudaSuccess) return cuda_error(e, "cudaEventCreate");
        if (g_plans.size() >= kMaxPlans) {   // evict the least recently used plan no graph holds
            for (size_t i = 0; i < g_plans.size(); ++i) {
                if (!g_plans[i]->captured) {
                    g_plans.erase(g_plans.begin() + static_cast<long>(i));
                    break;
                }
            }
        }
        g_plans.push_back(std::move(p));
        plan = g_plans.back().get();
    }

    auto fail = [&](cudaError_t err, const char* where) {
        char buf[160];
        if (pending != cudaSuccess)
            std::snprintf(buf, sizeof(buf), "%s (an earlier %s was pending on entry)", where, cudaGetErrorName(pending));
        else
            std::snprintf(buf, sizeof(buf), "%s", where);
        return cuda_error(err, buf);
    };
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(stream, &cap);
    if (e != cudaSuccess) return fail(e, "cudaStreamIsCapturing");
    const bool capturing = cap != cudaStreamCaptureStatusNone;
    if (capturing) plan->captured = true;
    cudaStream_t up = upload_stream ? upload_stream : stream;
    e = cudaMemsetAsync(workspace, 0, sizeof(unsigned), up);
    if (e != cudaSuccess) return fail(e, "status clear");
    if (plan->table_bytes) {
        e = cudaMemcpyAsync(plan->dev_tables, plan->pinned, plan->table_bytes, cudaMemcpyHostToDevice, up);
        if (e != cudaSuccess) return fail(e, "table upload");
    }
    if (before_launch) {
        const muon_status st = before_launch();
        if (st != MUON_OK) return st;
    }
    static const char* const kind_names[MUON_KERNEL_KINDS] = {"momentum", "scale", "ns_gemm", "update",
                                                              "simt_gemm", "lu", "misc", "tc_f32",
                                                              "simt_gemm_f64"};
    // NVTX: one range per launch, named by kernel kind, nested in one range for the call
    // (header-only NVTX 3: free unless a profiler injects its library)
    nvtxRangePushA("muon_b200 plan");
    struct RangeEnd {
        ~RangeEnd() { nvtxRangePop(); }
    } range_end;
    for (size_t si = 0; si < plan->steps.size(); ++si) {
        const PlanStep& s = plan->steps[si];
        nvtxRangePushA(s.kind >= 0 && s.kind < MUON_KERNEL_KINDS ? kind_names[s.kind] : "launch");
        struct LaunchRangeEnd {
            ~LaunchRangeEnd() { nvtxRangePop(); }
        } launch_range_end;
        if (g_timing.enabled) {
            TimingRec r{s.kind, s.work, nullptr, nullptr};
            cudaEventCreate(&r.e0);
            cudaEventCreate(&r.e1);
            cudaEventRecord(r.e0, stream);
            e = s.run(stream);
            cudaEventRecord(r.e1, stream);
            g_timing.pending.push_back(r);
        } else {
            e = s.run(stream);
        }
        if (e != cudaSuccess) {
            char buf[96];
            std::snprintf(buf, sizeof(buf), "launch %zu of %zu (%s)", si, plan->steps.size(),
                          s.kind >= 0 && s.kind < MUON_KERNEL_KINDS ? kind_names[s.kind] : "?");
            return fail(e, buf);
        }
    }
    if (!capturing) {
        e = cudaEventRecord(plan->last_use, stream);
        if (e != cudaSuccess) return fail(e, "cudaEventRecord");
        plan->recorded = true;
    }
    return MUON_OK;
}

void TmapPool::note_failure(const void* base, int rows, int cols, int box) {
    std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed for %p (%d x %d bf16, box %d)",
                  base, rows, cols, box);
}

bool encode_bf16_tmap(CUtensorMap* out, const void* base, int rows, int cols, int box_rows) {
    using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
    static EncodeFn fn = nullptr;
    if (fn == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || p == nullptr)
            return false;
        fn = reinterpret_cast<EncodeFn>(p);
    }
    const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(cols) * 2};
    const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estride[2] = {1u, 1u};
    const CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box,
                          estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace muon

extern "C" {

const char* muon_last_error(void) { return muon::g_last_error; }

muon_status muon_timing_enable(int enable) {
    std::lock_guard<std::mutex> lk(muon::g_mu);
    muon::g_timing.enabled = enable != 0;
    return MUON_OK;
}

muon_status muon_timing_reset(void) {
    std::lock_guard<std::mutex> lk(muon::g_mu);
    muon::drain_timing_locked();
    for (int k = 0; k < MUON_KERNEL_KINDS; ++k) {
        muon::g_timing.ms[k] = 0;
        muon::g_timing.launches[k] = 0;
        muon::g_timing.work[k] = 0;
    }
    return MUON_OK;
}

muon_status muon_timing_read(int kind, double* ms, long long* launches, double* work) {
    if (kind < 0 || kind >= MUON_KERNEL_KINDS || !ms || !launches || !work) return MUON_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(muon::g_mu);
    muon::drain_timing_locked();
    *ms = muon::g_timing.ms[kind];
    *launches = muon::g_timing.launches[kind];
    *work = muon::g_timing.work[kind];
    return MUON_OK;
}

}  // extern "C"
