// Host runtime shared by the entry points: workspace arena, device-table staging, the plan
// cache, kernel-kind timing and tensor-map encoding.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <functional>
#include <memory>
#include <string>
#include <vector>

#include "../../include/muon_b200.h"
#include "kernels.cuh"

namespace muon {

constexpr size_t kAlign = 256;
constexpr size_t kHeaderBytes = 256;   // device status word + padding at the workspace start

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Bump allocator over a device range (only offsets until `base` is known).
struct Arena {
    uint8_t* base = nullptr;
    size_t used = 0;
    size_t take(size_t bytes, size_t align = kAlign) {
        used = align_up(used, align);
        const size_t off = used;
        used += bytes;
        return off;
    }
    void* at(size_t off) const { return base ? base + off : nullptr; }
};

// Host image of the device tables of one plan.  Objects are appended with their final
// device address known (device base + offset), then the whole image is copied with one
// cudaMemcpyAsync from pinned memory.
struct TableImage {
    std::vector<uint8_t> bytes;
    uint8_t* dev_base = nullptr;  // device address of bytes[0]
    size_t add(const void* src, size_t n, size_t align) {
        size_t off = align_up(bytes.size(), align);
        bytes.resize(off + n);
        if (src) std::memcpy(bytes.data() + off, src, n);
        return off;
    }
    template <class T>
    T* dev(size_t off) const { return reinterpret_cast<T*>(dev_base + off); }
};

// One recorded launch of a plan: kind for timing, algorithmic work (FLOP or bytes).
struct PlanStep {
    int kind;
    double work;
    std::function<cudaError_t(cudaStream_t)> run;
};

struct Plan {
    std::vector<uint8_t> key;
    uint8_t* pinned = nullptr;       // host copy of the tables (pinned)
    size_t table_bytes = 0;
    uint8_t* dev_tables = nullptr;   // destination in the workspace
    std::vector<PlanStep> steps;
    cudaEvent_t last_use = nullptr;   // recorded after each run outside stream capture
    bool recorded = false;
    // Run at least once under stream capture: a graph may hold a copy node that reads
    // `pinned`, so the plan is never evicted.
    bool captured = false;
    ~Plan();
};

// Appends POD values to a cache key.
struct KeyWriter {
    std::vector<uint8_t> k;
    template <class T>
    void put(const T& v) {
        const uint8_t* p = reinterpret_cast<const uint8_t*>(&v);
        k.insert(k.end(), p, p + sizeof(T));
    }
    void put_bytes(const void* p, size_t n) {
        const uint8_t* q = static_cast<const uint8_t*>(p);
        k.insert(k.end(), q, q + n);
    }
};

// Finds a cached plan for `key` or builds one with `build` (which fills steps and the table
// image); then clears the workspace status word, copies the tables and runs the steps on
// `stream`.  With an `upload_stream` the status clear and the table copy go there instead,
// and `before_launch` (if set) runs after they are enqueued and before the first launch:
// it must order `stream` after the upload (an event).
muon_status run_plan(const std::vector<uint8_t>& key, void* workspace, size_t table_offset,
                     const std::function<muon_status(Plan&, TableImage&)>& build, cudaStream_t stream,
                     cudaStream_t upload_stream = nullptr,
                     const std::function<muon_status()>& before_launch = nullptr);

// Tensor map of a row-major bf16 matrix (rows x cols, pitch = cols) with a box of 64 columns
// x box_rows rows, 128-byte swizzle, zero fill out of bounds.
bool encode_bf16_tmap(CUtensorMap* out, const void* base, int rows, int cols, int box_rows);

// Tensor maps of one plan, deduplicated by (base, shape, box), stored in the table image.
struct TmapPool {
    TableImage& img;
    struct Entry {
        const void* base;
        int rows, cols, box;
        size_t off;
    };
    std::vector<Entry> entries;
    bool failed = false;
    explicit TmapPool(TableImage& i) : img(i) {}
    // Records the first failed encoding as the thread's last library error.
    void note_failure(const void* base, int rows, int cols, int box);
    const CUtensorMap* get(const void* base, int rows, int cols, int box) {
        if (base == nullptr) return nullptr;
        for (auto& e : entries)
            if (e.base == base && e.rows == rows && e.cols == cols && e.box == box) return img.dev<CUtensorMap>(e.off);
        CUtensorMap tm;
        if (!encode_bf16_tmap(&tm, base, rows, cols, box)) {
            if (!failed) note_failure(base, rows, cols, box);
            failed = true;
        }
        const size_t off = img.add(&tm, sizeof(tm), 128);
        entries.push_back({base, rows, cols, box, off});
        return img.dev<CUtensorMap>(off);
    }
};

int device_sm_count();
muon_status from_cuda(cudaError_t e);
// Records `where` and the CUDA error as the calling thread's last library error (read with
// muon_last_error) and returns MUON_ERR_CUDA.
muon_status cuda_error(cudaError_t e, const char* where);

}  // namespace muon
