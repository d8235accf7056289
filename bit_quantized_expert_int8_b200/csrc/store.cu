// store.cu -- the storage tier of the expert cache: expert blobs read from a
// file with parallel pread ("TurboFieldfare" article, daily.steinslab.io,
// "Trois optimisations clés" items 2 and 3: experts streamed from the SSD,
// read ahead with parallel pread; "Gemma 4 26B : Comment faire tourner un LLM
// en 2 Go de RAM", section 04 "Le pipeline de traitement" steps 3-4: only the
// missing experts are read).  Host code only.
//
// File: n_layers x n_experts blobs, layer-major, each padded to a multiple of
// 4096 bytes (moe_store_stride), so every read starts and ends on a 4 KiB
// boundary and O_DIRECT can bypass the page cache on any block size.  Reads
// are split into parts of at most kPart bytes and handed to a pool of
// threads, each issuing its own pread calls, into pinned staging buffers
// (page-aligned host memory when no GPU is present).
#include <fcntl.h>
#include <sys/stat.h>
#include <unistd.h>

#include <cerrno>
#include <cstdarg>
#include <chrono>
#include <condition_variable>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <deque>
#include <mutex>
#include <string>
#include <thread>
#include <vector>

#include <cuda_runtime.h>

#include "moeq4.h"

namespace {

constexpr size_t kAlign = 4096;
constexpr size_t kPart = 1u << 20;          // bytes per pread job

struct Job {
    off_t off;
    size_t len;
    uint8_t* dst;
};

}  // namespace

struct moe_store {
    int fd = -1;
    bool direct = false;
    int n_layers = 0, n_experts = 0;
    size_t blob = 0, stride = 0;
    std::vector<std::thread> threads;
    std::mutex mu;
    std::condition_variable cv_job, cv_done;
    std::deque<Job> q;
    int pending = 0;
    int err = 0;
    bool stop = false;
    uint8_t* staging = nullptr;
    bool staging_pinned = false;
    int n_staging = 0;
    unsigned long long bytes = 0;
    double seconds = 0.0;
};

// the library's per-thread error message (moe_last_error)
void moeq4_set_error(const char* msg);

static int store_fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    moeq4_set_error(buf);
    return code;
}

static void store_worker(moe_store* st) {
    for (;;) {
        Job j;
        {
            std::unique_lock<std::mutex> lk(st->mu);
            st->cv_job.wait(lk, [&] { return st->stop || !st->q.empty(); });
            if (st->stop && st->q.empty()) return;
            j = st->q.front();
            st->q.pop_front();
        }
        int e = 0;
        size_t done = 0;
        while (done < j.len) {
            const ssize_t r = pread(st->fd, j.dst + done, j.len - done, j.off + (off_t)done);
            if (r < 0) {
                if (errno == EINTR) continue;
                e = errno;
                break;
            }
            if (r == 0) { e = EIO; break; }    // the file ends early
            done += (size_t)r;
        }
        {
            std::lock_guard<std::mutex> lk(st->mu);
            if (e && !st->err) st->err = e;
            if (--st->pending == 0) st->cv_done.notify_all();
        }
    }
}

extern "C" size_t moe_store_stride(size_t blob_bytes) {
    return (blob_bytes + kAlign - 1) / kAlign * kAlign;
}

extern "C" int moe_store_close(moe_store* st) {
    if (!st) return MOE_OK;
    {
        std::lock_guard<std::mutex> lk(st->mu);
        st->stop = true;
    }
    st->cv_job.notify_all();
    for (auto& t : st->threads) t.join();
    if (st->fd >= 0) close(st->fd);
    if (st->staging) {
        if (st->staging_pinned) cudaFreeHost(st->staging);
        else free(st->staging);
    }
    delete st;
    return MOE_OK;
}

extern "C" int moe_store_open(const char* path, int n_layers, int n_experts, size_t blob_bytes,
                              int n_threads, int n_staging, moe_store** out) {
    if (!out) return store_fail(MOE_ERR_INVALID_ARG, "moe_store_open: out is NULL");
    *out = nullptr;
    if (!path || n_layers < 1 || n_experts < 1 || blob_bytes == 0 || blob_bytes % 16 ||
        n_threads < 1 || n_threads > 256 || n_staging < 1 || n_staging > 4096)
        return store_fail(MOE_ERR_INVALID_ARG, "moe_store_open: bad argument");
    moe_store* st = new moe_store();
    st->n_layers = n_layers;
    st->n_experts = n_experts;
    st->blob = blob_bytes;
    st->stride = moe_store_stride(blob_bytes);
    st->fd = open(path, O_RDONLY | O_DIRECT);
    st->direct = st->fd >= 0;
    if (st->fd < 0) st->fd = open(path, O_RDONLY);             // file systems without O_DIRECT
    if (st->fd < 0) {
        const int e = errno;
        delete st;
        return store_fail(MOE_ERR_INVALID_ARG, "moe_store_open: %s: %s", path, strerror(e));
    }
    struct stat sb{};
    const size_t need = (size_t)n_layers * n_experts * st->stride;
    if (fstat(st->fd, &sb) != 0 || (size_t)sb.st_size < need) {
        close(st->fd);
        delete st;
        return store_fail(MOE_ERR_INVALID_ARG, "moe_store_open: %s holds fewer than %zu bytes", path, need);
    }
    const size_t bytes = (size_t)n_staging * st->stride;
    void* p = nullptr;
    int dev_count = 0;
    if (cudaGetDeviceCount(&dev_count) == cudaSuccess && dev_count > 0 &&
        cudaHostAlloc(&p, bytes, cudaHostAllocDefault) == cudaSuccess) {
        st->staging_pinned = true;
    } else {
        cudaGetLastError();
        if (posix_memalign(&p, kAlign, bytes) != 0) p = nullptr;
    }
    if (!p) {
        close(st->fd);
        delete st;
        return store_fail(MOE_ERR_CUDA, "moe_store_open: cannot allocate %zu bytes of staging", bytes);
    }
    st->staging = static_cast<uint8_t*>(p);
    st->n_staging = n_staging;
    for (int i = 0; i < n_threads; i++) st->threads.emplace_back(store_worker, st);
    *out = st;
    return MOE_OK;
}

// Reads blobs (layer, experts[i]) into staging buffers i (i < n_staging),
// all in parallel; returns once every part is in.
static int store_read_staging(moe_store* st, int layer, const int32_t* experts, int n) {
    if (layer < 0 || layer >= st->n_layers || n < 0 || n > st->n_staging)
        return store_fail(MOE_ERR_INVALID_ARG, "moe_store_read: layer %d or count %d out of range", layer, n);
    for (int i = 0; i < n; i++)
        if (experts[i] < 0 || experts[i] >= st->n_experts)
            return store_fail(MOE_ERR_INVALID_ARG, "moe_store_read: expert %d out of range", experts[i]);
    const auto t0 = std::chrono::steady_clock::now();
    {
        std::lock_guard<std::mutex> lk(st->mu);
        st->err = 0;
        for (int i = 0; i < n; i++) {
            const off_t base = (off_t)(((size_t)layer * st->n_experts + experts[i]) * st->stride);
            uint8_t* dst = st->staging + (size_t)i * st->stride;
            for (size_t o = 0; o < st->stride; o += kPart) {
                st->q.push_back(Job{base + (off_t)o, st->stride - o < kPart ? st->stride - o : kPart, dst + o});
                st->pending++;
            }
        }
    }
    st->cv_job.notify_all();
    int err;
    {
        std::unique_lock<std::mutex> lk(st->mu);
        st->cv_done.wait(lk, [&] { return st->pending == 0; });
        err = st->err;
    }
    st->seconds += std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count();
    st->bytes += (unsigned long long)n * st->blob;
    if (err) return store_fail(MOE_ERR_CACHE_STATE, "moe_store_read: %s", strerror(err));
    return MOE_OK;
}

extern "C" int moe_store_read(moe_store* st, int layer, const int32_t* experts, int n, void* const* dst) {
    if (!st || (n > 0 && (!experts || !dst)))
        return store_fail(MOE_ERR_INVALID_ARG, "moe_store_read: NULL argument");
    for (int done = 0; done < n;) {
        const int m = n - done < st->n_staging ? n - done : st->n_staging;
        const int rc = store_read_staging(st, layer, experts + done, m);
        if (rc != MOE_OK) return rc;
        for (int i = 0; i < m; i++) memcpy(dst[done + i], st->staging + (size_t)i * st->stride, st->blob);
        done += m;
    }
    return MOE_OK;
}

extern "C" int moe_store_stats(const moe_store* st, unsigned long long* bytes, double* seconds, int* direct) {
    if (!st) return store_fail(MOE_ERR_INVALID_ARG, "moe_store_stats: NULL store");
    if (bytes) *bytes = st->bytes;
    if (seconds) *seconds = st->seconds;
    if (direct) *direct = st->direct ? 1 : 0;
    return MOE_OK;
}

// Library-internal: fill cache slots from the store.  Reads the blobs of
// experts[0..n) of `layer` (at most n_staging at a time) and copies each into
// slots + slot[i] * blob on `copy` (after the previous batch's copies, which
// read the same staging buffers).  `copy_done` is recorded on `copy` after
// the last copy.
int moeq4_store_fill(moe_store* st, int layer, const int32_t* experts, const int32_t* slot, int n,
                     uint8_t* slots, cudaStream_t copy, cudaEvent_t copy_done) {
    for (int done = 0; done < n;) {
        const int m = n - done < st->n_staging ? n - done : st->n_staging;
        // the staging buffers are free once the earlier copies out of them ended
        cudaError_t e = cudaEventSynchronize(copy_done);
        if (e != cudaSuccess) return store_fail(MOE_ERR_CUDA, "store fill: %s", cudaGetErrorString(e));
        const int rc = store_read_staging(st, layer, experts + done, m);
        if (rc != MOE_OK) return rc;
        for (int i = 0; i < m; i++) {
            e = cudaMemcpyAsync(slots + (size_t)slot[done + i] * st->blob, st->staging + (size_t)i * st->stride,
                                st->blob, cudaMemcpyHostToDevice, copy);
            if (e != cudaSuccess) return store_fail(MOE_ERR_CUDA, "store fill copy: %s", cudaGetErrorString(e));
        }
        e = cudaEventRecord(copy_done, copy);
        if (e != cudaSuccess) return store_fail(MOE_ERR_CUDA, "store fill: %s", cudaGetErrorString(e));
        done += m;
    }
    return MOE_OK;
}

size_t moeq4_store_blob(const moe_store* st) { return st->blob; }
