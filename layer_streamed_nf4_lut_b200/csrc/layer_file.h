// File-backed NF4 layer stack: the "stream from disk" source for stacks larger than host RAM
// (rug.gal radar "Soup ... layer streaming", "En detalle": the base lives in CPU RAM or on
// disk; imasters "Como cabe um 8B em 4 GB": stream_source auto = RAM when it fits, else NVMe).
//
// Layout: layer i occupies [i * stride, i * stride + blob_bytes) of one file, stride =
// blob_bytes rounded up to 4096 (page-aligned reads).  A reader thread fills a ring of
// page-locked staging slots in request order; the copy stream runs, per layer load,
//   host func "wait until request s is read"  ->  cudaMemcpyAsync(slot -> device buffer)
//   ->  host func "slot of request s is free again".
// Requests and stream operations are issued in the same order, so a slot is always released
// (by an earlier host func of the same stream) before the reader needs it again.  Every wait
// is bounded; a failed or short read, or a wait that runs out, sets an error the next step
// reports as SOUP_ERR_IO.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <condition_variable>
#include <deque>
#include <mutex>
#include <string>
#include <thread>
#include <vector>

namespace soup {

class LayerFile {
 public:
  LayerFile() = default;
  ~LayerFile() { close(); }
  LayerFile(const LayerFile&) = delete;
  LayerFile& operator=(const LayerFile&) = delete;

  // Creates (or truncates) the file, sizes it to n_layers * stride, allocates n_slots pinned
  // staging slots and starts the reader thread.  wait_ms bounds every wait.
  bool open(const std::string& path, int n_layers, size_t blob_bytes, int n_slots, long long wait_ms,
            std::string& err);
  void close();
  bool is_open() const { return fd_ >= 0; }

  // Synchronous whole-blob write / read (quantiser output, user loads and reads).
  bool write(int layer, const void* src, std::string& err);
  bool read(int layer, void* dst, std::string& err);

  // Queues an asynchronous read of `layer` into the next staging slot and enqueues on
  // `copy_stream`: wait for that read, copy the slot to `dst` (blob_bytes), release the slot.
  cudaError_t stream_layer(int layer, void* dst, cudaStream_t copy_stream);

  // A pinned blob-sized buffer (slot 0) for link probes; valid while open.
  uint8_t* probe_buffer() const { return slots_.empty() ? nullptr : slots_[0]; }

  // First error since the last call (empty if none); clears it.
  std::string take_error();
  size_t stride() const { return stride_; }
  long long bytes_read() const;
  double read_ms() const;

 private:
  struct Req {
    long long seq;
    int layer;
  };
  struct Arg {
    LayerFile* f;
    long long seq;
  };
  static void CUDART_CB host_wait_read(void* arg);
  static void CUDART_CB host_release(void* arg);
  void reader_loop();
  bool pread_all(void* dst, size_t bytes, long long off, std::string& err);
  void set_error(const std::string& e);

  int fd_ = -1;
  int n_layers_ = 0;
  size_t blob_ = 0, stride_ = 0;
  long long wait_ms_ = 600000;
  std::vector<uint8_t*> slots_;

  std::thread reader_;
  mutable std::mutex mu_;
  std::condition_variable cv_req_, cv_ready_, cv_free_;
  std::deque<Req> queue_;
  long long next_seq_ = 0;
  long long ready_seq_ = -1;          // requests read so far (in order)
  std::vector<long long> released_;   // per slot: last request whose copy has finished
  bool stop_ = false;
  std::string error_;
  long long bytes_read_ = 0;
  double read_ms_ = 0.0;
};

}  // namespace soup
