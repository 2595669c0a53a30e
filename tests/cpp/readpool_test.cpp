// CPU test of the file store's reader pool (csrc/readpool.h) with a stub in
// place of pread: one descriptor whose read blocks until the test releases it
// (a slow device), one that fails, one whose file is short.  Built with the
// address and undefined-behaviour sanitizers by tests/test_readpool.py.
#include <cerrno>
#include <condition_variable>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <thread>
#include <vector>

#include "readpool.h"

using moe::ReadPool;

static std::mutex g_mu;
static std::condition_variable g_cv;
static bool g_release = false;

enum { kFast = 1, kSlow = 2, kBroken = 3, kShort = 4, kCounted = 5 };
static int g_counted = 0;

static ssize_t stub_pread(int fd, void* dst, size_t len, off_t off) {
    if (fd == kSlow) {
        std::unique_lock<std::mutex> lock(g_mu);
        g_cv.wait(lock, [] { return g_release; });
    }
    if (fd == kCounted) {
        std::lock_guard<std::mutex> lock(g_mu);
        ++g_counted;
    }
    if (fd == kBroken) {
        errno = EIO;
        return -1;
    }
    if (fd == kShort) {
        if (off >= 100) return 0;
        if (len > size_t(100 - off)) len = size_t(100 - off);
    }
    std::memset(dst, fd, len);
    return ssize_t(len);
}

#define CHECK(c)                                                        \
    do {                                                                \
        if (!(c)) {                                                     \
            std::printf("FAILED line %d: %s\n", __LINE__, #c);           \
            std::exit(1);                                               \
        }                                                               \
    } while (0)

int main() {
    ReadPool pool(2, stub_pread);
    std::vector<std::vector<unsigned char>> bufs(5, std::vector<unsigned char>(4096, 0));
    auto job = [&](int fd, int buf, size_t len, size_t need) {
        ReadPool::Job j;
        j.fd = fd;
        j.offset = 0;
        j.len = len;
        j.need = need;
        j.dst = bufs[size_t(buf)].data();
        return j;
    };
    // 1. a normal batch
    CHECK(pool.begin_batch(2));
    pool.submit(0, job(kFast, 0, 4096, 4096));
    pool.submit(1, job(kFast, 1, 4096, 4096));
    CHECK(pool.wait(0, 2000) == ReadPool::kDone);
    CHECK(pool.wait(1, 2000) == ReadPool::kDone);
    CHECK(bufs[0][4095] == kFast && bufs[1][0] == kFast);

    // 2. a read that outlasts the caller's limit: the batch is abandoned with
    //    the read still running in its thread
    CHECK(pool.begin_batch(3));
    pool.submit(0, job(kFast, 0, 4096, 4096));
    pool.submit(1, job(kSlow, 1, 4096, 4096));
    pool.submit(2, job(kFast, 2, 4096, 4096));
    CHECK(pool.wait(0, 2000) == ReadPool::kDone);
    CHECK(pool.wait(1, 50) == ReadPool::kPending);  // timed out
    CHECK(!pool.abandon(50));                         // still running
    CHECK(pool.running() == 1);

    // 3. no new batch while that read may still write its buffer
    CHECK(!pool.begin_batch(1));

    // 4. the slow read finishes; then a larger batch (the job table grows)
    //    runs normally, and the straggler's late result went nowhere else
    {
        std::lock_guard<std::mutex> lock(g_mu);
        g_release = true;
    }
    g_cv.notify_all();
    for (int i = 0; i < 400 && pool.running() > 0; ++i) std::this_thread::sleep_for(std::chrono::milliseconds(5));
    CHECK(pool.running() == 0);
    CHECK(bufs[1][0] == kSlow);
    CHECK(pool.begin_batch(5));
    for (int i = 0; i < 5; ++i) pool.submit(i, job(kFast, i, 4096, 4096));
    for (int i = 0; i < 5; ++i) CHECK(pool.wait(i, 2000) == ReadPool::kDone);

    // 5. a failing read and a short file are failures; a short read that
    //    still covers what must exist is not
    CHECK(pool.begin_batch(3));
    pool.submit(0, job(kBroken, 0, 4096, 4096));
    pool.submit(1, job(kShort, 1, 4096, 4096));
    pool.submit(2, job(kShort, 2, 4096, 100));
    CHECK(pool.wait(0, 2000) == ReadPool::kFailed);
    CHECK(pool.wait(1, 2000) == ReadPool::kFailed);
    CHECK(pool.wait(2, 2000) == ReadPool::kDone);
    CHECK(pool.abandon(2000));

    // 6. a batch abandoned after a failure while reads are still queued and
    //    running: the queued one is cancelled and never runs, the running
    //    ones end once released, and the pool is usable again
    {
        std::lock_guard<std::mutex> lock(g_mu);
        g_release = false;
    }
    g_counted = 0;
    CHECK(pool.begin_batch(4));
    pool.submit(0, job(kBroken, 0, 4096, 4096));
    pool.submit(1, job(kSlow, 1, 4096, 4096));
    pool.submit(2, job(kSlow, 2, 4096, 4096));
    pool.submit(3, job(kCounted, 3, 4096, 4096));
    CHECK(pool.wait(0, 2000) == ReadPool::kFailed);
    pool.abandon(50);
    {
        std::lock_guard<std::mutex> lock(g_mu);
        g_release = true;
    }
    g_cv.notify_all();
    for (int i = 0; i < 400 && pool.running() > 0; ++i) std::this_thread::sleep_for(std::chrono::milliseconds(5));
    CHECK(pool.running() == 0);
    CHECK(g_counted == 0);
    CHECK(pool.begin_batch(1));
    pool.submit(0, job(kCounted, 4, 4096, 4096));
    CHECK(pool.wait(0, 2000) == ReadPool::kDone && g_counted == 1);
    std::printf("readpool ok\n");
    return 0;
}
