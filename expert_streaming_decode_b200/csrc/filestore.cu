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
// has completed.  The reader threads and their failure handling are in
// readpool.h.  Host code only.
#include <unistd.h>

#include "filestore.cuh"
#include "readpool.h"

namespace moe {

namespace {
constexpr int kReadThreads = 4;  // reads in flight (bounded parallelism)
}

FileReader::~FileReader() {
    delete pool_;  // joins the reader threads
    for (auto e : events_) cudaEventDestroy(e);
    for (auto b : bufs_) cudaFreeHost(b);
}

int FileReader::ensure(size_t buf_bytes, int nbuf) {
    if (pool_ && buf_bytes <= buf_bytes_ && int(bufs_.size()) >= nbuf) return MOE_OK;
    if (pool_) return MOE_ERR_STATE;  // sized once per context
    for (int i = 0; i < nbuf; ++i) {
        void* p = nullptr;
        if (cudaHostAlloc(&p, buf_bytes, cudaHostAllocDefault) != cudaSuccess) return MOE_ERR_CUDA;
        bufs_.push_back(static_cast<uint8_t*>(p));
        cudaEvent_t e;
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return MOE_ERR_CUDA;
        events_.push_back(e);
    }
    buf_bytes_ = buf_bytes;
    pool_ = new ReadPool(kReadThreads, [](int fd, void* dst, size_t len, off_t off) { return pread(fd, dst, len, off); });
    return MOE_OK;
}

int FileReader::read_and_copy(const std::vector<FileRead>& reads, cudaStream_t side, int timeout_ms,
                              uint64_t* bytes) {
    const int n = int(reads.size()), nbuf = int(bufs_.size());
    if (n == 0) return MOE_OK;
    if (!pool_ || nbuf == 0) return MOE_ERR_STATE;
    for (const auto& r : reads)
        if (r.len > buf_bytes_ || r.need > r.len) return MOE_ERR_ARG;
    // refused while a read of an abandoned earlier batch still writes a buffer
    if (!pool_->begin_batch(n)) return MOE_ERR_STATE;
    auto submit = [&](int i) {
        ReadPool::Job j;
        j.fd = reads[i].fd;
        j.offset = reads[i].offset;
        j.len = reads[i].len;
        j.need = reads[i].need;
        j.dst = bufs_[i % nbuf];
        pool_->submit(i, j);
    };
    // a buffer's previous copy (an earlier call) must be complete before it is refilled
    for (int b = 0; b < nbuf && b < n; ++b)
        if (cudaEventSynchronize(events_[b]) != cudaSuccess) return MOE_ERR_CUDA;
    for (int i = 0; i < n && i < nbuf; ++i) submit(i);
    int rc = MOE_OK;
    for (int i = 0; i < n; ++i) {
        const int st = pool_->wait(i, timeout_ms);
        if (st == ReadPool::kPending) { rc = MOE_ERR_TIMEOUT; break; }
        if (st != ReadPool::kDone) { rc = MOE_ERR_IO; break; }
        const int b = i % nbuf;
        if (cudaMemcpyAsync(reads[i].dst, bufs_[b], reads[i].need, cudaMemcpyHostToDevice, side) != cudaSuccess ||
            cudaEventRecord(events_[b], side) != cudaSuccess) {
            rc = MOE_ERR_CUDA;
            break;
        }
        *bytes += reads[i].need;
        if (i + nbuf < n) {
            // buffer b is next filled by read i + nbuf, once this copy has landed
            if (cudaEventSynchronize(events_[b]) != cudaSuccess) { rc = MOE_ERR_CUDA; break; }
            submit(i + nbuf);
        }
    }
    // on failure: cancel what is queued, wait (bounded) for reads in progress;
    // any still running keep the pool closed to new batches until they end
    if (rc != MOE_OK) pool_->abandon(timeout_ms);
    return rc;
}

}  // namespace moe
