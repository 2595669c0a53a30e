// readpool.h -- the bounded-parallel positional reader behind the file-backed
// expert store (filestore.cu): a few threads take read jobs from a queue, each
// job reads one missed expert from a file into a host buffer.  Host-only C++,
// no CUDA, so its failure handling can be tested on a CPU.
//
// Method: misses are read with several positional reads in flight, not through
// a memory map ("Gemma 4 26B en ~2 GB de RAM ...", section "Por que pread y no
// mmap"; "TurboFieldfare: motor open source ...", section "Proceso de
// generacion de tokens": bounded parallel reads).
//
// Failure handling.  A batch that fails (a read error, or a read that takes
// longer than the caller's limit) is abandoned: queued jobs are cancelled, and
// the caller waits a bounded time for the jobs a thread has already started.
// A job still running after that (a straggler) keeps writing into its buffer,
// so the pool refuses new batches (begin_batch returns false) until every
// straggler has finished; a straggler's result is dropped, because each batch
// has its own generation number and a job only reports into the batch it was
// started for.
#pragma once

#include <sys/types.h>

#include <cerrno>
#include <chrono>
#include <condition_variable>
#include <cstddef>
#include <cstdint>
#include <deque>
#include <functional>
#include <mutex>
#include <thread>
#include <vector>

namespace moe {

class ReadPool {
public:
    // positional read: like pread(2), returns bytes read, 0 at end of file,
    // -1 with errno set on error
    using ReadFn = std::function<ssize_t(int fd, void* dst, size_t len, off_t offset)>;
    enum Status : int { kPending = 0, kDone = 1, kFailed = -1, kCancelled = -2 };
    struct Job {
        int fd = -1;
        uint64_t offset = 0;
        size_t len = 0, need = 0;  // bytes to read, bytes that must exist
        void* dst = nullptr;
    };

    ReadPool(int threads, ReadFn fn) : read_(std::move(fn)) {
        for (int t = 0; t < threads; ++t) threads_.emplace_back([this] { worker(); });
    }
    ~ReadPool() {
        {
            std::lock_guard<std::mutex> lock(mu_);
            stop_ = true;
            queue_.clear();
        }
        cv_work_.notify_all();
        for (auto& t : threads_) t.join();
    }
    ReadPool(const ReadPool&) = delete;
    ReadPool& operator=(const ReadPool&) = delete;

    // Starts a batch of n jobs.  False while a job of an abandoned batch is
    // still running (its buffer is still being written).
    bool begin_batch(int n) {
        std::lock_guard<std::mutex> lock(mu_);
        if (running_ > 0) return false;
        ++gen_;
        queue_.clear();
        jobs_.assign(size_t(n), Slot{});
        return true;
    }
    void submit(int i, const Job& j) {
        {
            std::lock_guard<std::mutex> lock(mu_);
            jobs_[size_t(i)].job = j;
            jobs_[size_t(i)].status = kPending;
            jobs_[size_t(i)].submitted = true;
            queue_.push_back(i);
        }
        cv_work_.notify_one();
    }
    // Waits up to timeout_ms for job i: kDone, kFailed, or kPending (timed out).
    int wait(int i, int timeout_ms) {
        std::unique_lock<std::mutex> lock(mu_);
        cv_done_.wait_for(lock, std::chrono::milliseconds(timeout_ms),
                          [&] { return jobs_[size_t(i)].status != kPending; });
        return jobs_[size_t(i)].status;
    }
    // Abandons the batch: cancels the queued jobs and waits up to timeout_ms
    // for the started ones.  True when none is left running.
    bool abandon(int timeout_ms) {
        std::unique_lock<std::mutex> lock(mu_);
        for (int j : queue_) jobs_[size_t(j)].status = kCancelled;
        queue_.clear();
        cv_done_.wait_for(lock, std::chrono::milliseconds(timeout_ms), [&] { return running_ == 0; });
        return running_ == 0;
    }
    // Jobs a thread is executing now (stragglers after an abandoned batch).
    int running() {
        std::lock_guard<std::mutex> lock(mu_);
        return running_;
    }

private:
    struct Slot {
        Job job;
        int status = kPending;
        bool submitted = false;
    };
    void worker() {
        for (;;) {
            Job job;
            int idx;
            uint64_t gen;
            {
                std::unique_lock<std::mutex> lock(mu_);
                cv_work_.wait(lock, [&] { return stop_ || !queue_.empty(); });
                if (stop_) return;
                idx = queue_.front();
                queue_.pop_front();
                job = jobs_[size_t(idx)].job;
                gen = gen_;
                ++running_;
            }
            size_t got = 0;
            int st = kDone;
            uint8_t* dst = static_cast<uint8_t*>(job.dst);
            while (got < job.len) {
                const ssize_t r = read_(job.fd, dst + got, job.len - got, off_t(job.offset + got));
                if (r < 0) {
                    if (errno == EINTR) continue;
                    st = kFailed;
                    break;
                }
                if (r == 0) break;  // end of file
                got += size_t(r);
            }
            if (st == kDone && got < job.need) st = kFailed;  // the blob itself must be complete
            {
                std::lock_guard<std::mutex> lock(mu_);
                // only into the batch the job was started for
                if (gen == gen_ && size_t(idx) < jobs_.size()) jobs_[size_t(idx)].status = st;
                --running_;
            }
            cv_done_.notify_all();
        }
    }

    ReadFn read_;
    std::mutex mu_;
    std::condition_variable cv_work_, cv_done_;
    std::deque<int> queue_;
    std::vector<Slot> jobs_;
    std::vector<std::thread> threads_;
    uint64_t gen_ = 0;
    int running_ = 0;
    bool stop_ = false;
};

}  // namespace moe
