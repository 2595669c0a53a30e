// filestore.cu -- the file-backed expert store: misses read with bounded
// parallel pread into pinned staging buffers, then copied to their slots.
//
// Method: the experts live on storage and a miss is read with several
// positional reads in flight instead of a memory map ("Gemma 4 26B en ~2 GB
// de RAM ...", section "Por que pread y no mmap"; "TurboFieldfare: motor open
// source ...", section "Proceso de generacion de tokens": misses are filled by
// bounded parallel reads).  Here the reads land in page-aligned pinned host
// buffers, so a file opened with O_DIRECT bypasses the page cache, and each
// buffer is copied to its HBM slot by cudaMemcpyAsync on the context's side
// stream as soon as its read is done; a buffer is reused only after its copy
// has completed.  Host code only.
#include <cerrno>
#include <chrono>
#include <condition_variable>
#include <deque>
#include <mutex>
#include <thread>
#include <vector>

#include <unistd.h>

#include "filestore.cuh"

namespace moe {

namespace {
constexpr int kReadThreads = 4;  // reads in flight (bounded parallelism)
}

struct FileReader::Impl {
    struct Job {
        int fd = -1;
        uint64_t offset = 0;
        size_t len = 0, need = 0;
        int buf = 0;
        int status = 0;  // 0 pending, 1 done, -1 failed, -2 cancelled
    };
    std::mutex mu;
    std::condition_variable cv_work, cv_done;
    std::deque<int> queue;     // indices into jobs
    std::vector<Job> jobs;
    std::vector<std::thread> threads;
    bool stop = false;

    void worker(std::vector<uint8_t*>* bufs) {
        for (;;) {
            int j;
            {
                std::unique_lock<std::mutex> lock(mu);
                cv_work.wait(lock, [&] { return stop || !queue.empty(); });
                if (stop && queue.empty()) return;
                j = queue.front();
                queue.pop_front();
            }
            Job job;
            {
                std::lock_guard<std::mutex> lock(mu);
                job = jobs[j];
            }
            uint8_t* dst = (*bufs)[job.buf];
            size_t got = 0;
            int st = 1;
            while (got < job.len) {
                const ssize_t r = pread(job.fd, dst + got, job.len - got, off_t(job.offset + got));
                if (r < 0) {
                    if (errno == EINTR) continue;
                    st = -1;
                    break;
                }
                if (r == 0) break;  // end of file
                got += size_t(r);
            }
            if (got < job.need) st = -1;  // the blob itself must be complete
            {
                std::lock_guard<std::mutex> lock(mu);
                jobs[j].status = st;
            }
            cv_done.notify_all();
        }
    }
};

FileReader::~FileReader() {
    if (impl_) {
        {
            std::lock_guard<std::mutex> lock(impl_->mu);
            impl_->stop = true;
        }
        impl_->cv_work.notify_all();
        for (auto& t : impl_->threads) t.join();
        delete impl_;
    }
    for (auto e : events_) cudaEventDestroy(e);
    for (auto b : bufs_) cudaFreeHost(b);
}

int FileReader::ensure(size_t buf_bytes, int nbuf) {
    if (impl_ && buf_bytes <= buf_bytes_ && int(bufs_.size()) >= nbuf) return MOE_OK;
    if (impl_) return MOE_ERR_STATE;  // sized once per context
    for (int i = 0; i < nbuf; ++i) {
        void* p = nullptr;
        if (cudaHostAlloc(&p, buf_bytes, cudaHostAllocDefault) != cudaSuccess) return MOE_ERR_CUDA;
        bufs_.push_back(static_cast<uint8_t*>(p));
        cudaEvent_t e;
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return MOE_ERR_CUDA;
        events_.push_back(e);
    }
    buf_bytes_ = buf_bytes;
    impl_ = new Impl();
    for (int t = 0; t < kReadThreads; ++t) impl_->threads.emplace_back([this] { impl_->worker(&bufs_); });
    return MOE_OK;
}

int FileReader::read_and_copy(const std::vector<FileRead>& reads, cudaStream_t side, int timeout_ms,
                              uint64_t* bytes) {
    const int n = int(reads.size()), nbuf = int(bufs_.size());
    if (n == 0) return MOE_OK;
    if (!impl_ || nbuf == 0) return MOE_ERR_STATE;
    for (const auto& r : reads)
        if (r.len > buf_bytes_ || r.need > r.len) return MOE_ERR_ARG;
    auto submit = [&](int i) {
        std::lock_guard<std::mutex> lock(impl_->mu);
        Impl::Job job;
        job.fd = reads[i].fd;
        job.offset = reads[i].offset;
        job.len = reads[i].len;
        job.need = reads[i].need;
        job.buf = i % nbuf;
        impl_->jobs[i] = job;
        impl_->queue.push_back(i);
    };
    {
        std::lock_guard<std::mutex> lock(impl_->mu);
        impl_->jobs.assign(n, Impl::Job{});
        impl_->queue.clear();
    }
    // a buffer's previous copy (an earlier call) must be complete before it is refilled
    for (int b = 0; b < nbuf && b < n; ++b)
        if (cudaEventSynchronize(events_[b]) != cudaSuccess) return MOE_ERR_CUDA;
    for (int i = 0; i < n && i < nbuf; ++i) submit(i);
    impl_->cv_work.notify_all();
    int rc = MOE_OK;
    int done_through = 0;
    for (int i = 0; i < n; ++i) {
        int st;
        {
            std::unique_lock<std::mutex> lock(impl_->mu);
            const bool ok = impl_->cv_done.wait_for(lock, std::chrono::milliseconds(timeout_ms),
                                                    [&] { return impl_->jobs[i].status != 0; });
            st = ok ? impl_->jobs[i].status : 0;
        }
        if (st == 0) { rc = MOE_ERR_TIMEOUT; break; }
        if (st < 0) { rc = MOE_ERR_IO; break; }
        const int b = i % nbuf;
        if (cudaMemcpyAsync(reads[i].dst, bufs_[b], reads[i].need, cudaMemcpyHostToDevice, side) != cudaSuccess ||
            cudaEventRecord(events_[b], side) != cudaSuccess) {
            rc = MOE_ERR_CUDA;
            break;
        }
        *bytes += reads[i].need;
        done_through = i + 1;
        if (i + nbuf < n) {
            // buffer b is next filled by read i + nbuf, once this copy has landed
            if (cudaEventSynchronize(events_[b]) != cudaSuccess) { rc = MOE_ERR_CUDA; break; }
            submit(i + nbuf);
            impl_->cv_work.notify_one();
        }
    }
    if (rc != MOE_OK) {
        // before the buffers can be reused: cancel the reads still queued and
        // wait (bounded) for the ones a worker has already started
        std::unique_lock<std::mutex> lock(impl_->mu);
        for (int j : impl_->queue) impl_->jobs[j].status = -2;
        impl_->queue.clear();
        for (int i = done_through; i < n; ++i) {
            if (impl_->jobs[i].fd < 0) continue;  // never submitted
            impl_->cv_done.wait_for(lock, std::chrono::milliseconds(timeout_ms),
                                    [&] { return impl_->jobs[i].status != 0; });
        }
    }
    return rc;
}

}  // namespace moe
