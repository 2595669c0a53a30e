// filestore.cuh -- host interface of the file-backed expert store (filestore.cu).
#pragma once
#include <cstddef>
#include <cstdint>
#include <vector>

#include <cuda_runtime.h>

#include "moe.h"

namespace moe {

class ReadPool;

// One miss: read [offset, offset + len) of fd (at least `need` bytes must
// exist) and copy the first `need` bytes to the device address dst.
struct FileRead {
    int fd;
    uint64_t offset;
    size_t len, need;
    uint8_t* dst;
};

// Pinned staging buffers plus a small pool of reader threads, owned by a
// context.  Not thread-safe: one call at a time (the context's contract).
class FileReader {
public:
    FileReader() = default;
    ~FileReader();
    FileReader(const FileReader&) = delete;
    FileReader& operator=(const FileReader&) = delete;
    // allocates nbuf page-aligned pinned buffers of buf_bytes and starts the
    // reader threads (first call only; later calls must fit)
    int ensure(size_t buf_bytes, int nbuf);
    // reads every entry with up to `buffers` reads in flight and issues its
    // copy on `side` as soon as it is read; returns MOE_OK, MOE_ERR_IO (read
    // failed or file too short), MOE_ERR_TIMEOUT (a read took longer than
    // timeout_ms), MOE_ERR_STATE (a read of an earlier failed call is still
    // running: its buffer is not free yet) or MOE_ERR_CUDA.  Adds the copied
    // bytes to *bytes.
    int read_and_copy(const std::vector<FileRead>& reads, cudaStream_t side, int timeout_ms, uint64_t* bytes);

private:
    ReadPool* pool_ = nullptr;
    std::vector<uint8_t*> bufs_;
    std::vector<cudaEvent_t> events_;
    size_t buf_bytes_ = 0;
};

}  // namespace moe
