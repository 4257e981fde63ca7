// File-backed NF4 layer stack (host code): see layer_file.h.
#include "layer_file.h"

#include <fcntl.h>
#include <sys/stat.h>
#include <unistd.h>

#include <cerrno>
#include <chrono>
#include <cstring>

namespace soup {

namespace {
constexpr size_t PAGE = 4096;
constexpr int READ_THREADS = 4;  // parallel chunks of one layer read
}  // namespace

bool LayerFile::open(const std::string& path, int n_layers, size_t blob_bytes, int n_slots, long long wait_ms,
                     std::string& err) {
  close();
  if (n_layers < 1 || blob_bytes == 0 || n_slots < 1) {
    err = "layer file: bad sizes";
    return false;
  }
  n_layers_ = n_layers;
  blob_ = blob_bytes;
  stride_ = (blob_bytes + PAGE - 1) / PAGE * PAGE;
  wait_ms_ = wait_ms > 0 ? wait_ms : 600000;
  fd_ = ::open(path.c_str(), O_RDWR | O_CREAT | O_TRUNC, 0644);
  if (fd_ < 0) {
    err = "layer file: open " + path + ": " + std::strerror(errno);
    return false;
  }
  if (::ftruncate(fd_, static_cast<off_t>(stride_) * n_layers) != 0) {
    err = "layer file: size " + path + ": " + std::strerror(errno);
    close();
    return false;
  }
  for (int k = 0; k < n_slots; ++k) {
    void* p = nullptr;
    if (cudaHostAlloc(&p, blob_, cudaHostAllocDefault) != cudaSuccess) {
      err = "layer file: pinned staging allocation failed";
      close();
      return false;
    }
    slots_.push_back(static_cast<uint8_t*>(p));
  }
  released_.assign(n_slots, 0);
  for (int k = 0; k < n_slots; ++k) released_[k] = static_cast<long long>(k) - n_slots;  // all free
  next_seq_ = 0;
  ready_seq_ = -1;
  stop_ = false;
  error_.clear();
  reader_ = std::thread([this] { reader_loop(); });
  return true;
}

void LayerFile::close() {
  if (reader_.joinable()) {
    {
      std::lock_guard<std::mutex> lk(mu_);
      stop_ = true;
    }
    cv_req_.notify_all();
    cv_free_.notify_all();
    cv_ready_.notify_all();
    reader_.join();
  }
  for (uint8_t* p : slots_) cudaFreeHost(p);
  slots_.clear();
  queue_.clear();
  if (fd_ >= 0) ::close(fd_);
  fd_ = -1;
}

bool LayerFile::pread_all(void* dst, size_t bytes, long long off, std::string& err) {
  // READ_THREADS page-aligned chunks in parallel (a single stream of reads leaves NVMe queues
  // and the page-cache copy under-used)
  const size_t chunk = ((bytes + READ_THREADS - 1) / READ_THREADS + PAGE - 1) / PAGE * PAGE;
  std::vector<std::thread> th;
  std::vector<int> ok(READ_THREADS, 1);
  for (int t = 0; t < READ_THREADS; ++t) {
    const size_t lo = static_cast<size_t>(t) * chunk;
    if (lo >= bytes) break;
    const size_t n = std::min(chunk, bytes - lo);
    th.emplace_back([&, t, lo, n] {
      size_t done = 0;
      while (done < n) {
        const ssize_t r = ::pread(fd_, static_cast<uint8_t*>(dst) + lo + done, n - done,
                                  static_cast<off_t>(off + lo + done));
        if (r < 0 && errno == EINTR) continue;
        if (r <= 0) {
          ok[t] = 0;
          return;
        }
        done += static_cast<size_t>(r);
      }
    });
  }
  for (auto& x : th) x.join();
  for (int t = 0; t < READ_THREADS; ++t)
    if (!ok[t]) {
      err = "layer file: short or failed read";
      return false;
    }
  return true;
}

bool LayerFile::write(int layer, const void* src, std::string& err) {
  if (fd_ < 0 || layer < 0 || layer >= n_layers_) {
    err = "layer file: not open or bad layer";
    return false;
  }
  size_t done = 0;
  const long long off = static_cast<long long>(layer) * stride_;
  while (done < blob_) {
    const ssize_t r = ::pwrite(fd_, static_cast<const uint8_t*>(src) + done, blob_ - done,
                               static_cast<off_t>(off + done));
    if (r < 0 && errno == EINTR) continue;
    if (r <= 0) {
      err = std::string("layer file: write: ") + std::strerror(errno);
      return false;
    }
    done += static_cast<size_t>(r);
  }
  // the stack is meant for sizes host RAM cannot hold: write it through and keep it out of the
  // page cache, so later reads come from the device, not from cached pages
  ::fdatasync(fd_);
  ::posix_fadvise(fd_, static_cast<off_t>(off), static_cast<off_t>(stride_), POSIX_FADV_DONTNEED);
  return true;
}

bool LayerFile::read(int layer, void* dst, std::string& err) {
  if (fd_ < 0 || layer < 0 || layer >= n_layers_) {
    err = "layer file: not open or bad layer";
    return false;
  }
  return pread_all(dst, blob_, static_cast<long long>(layer) * stride_, err);
}

void LayerFile::set_error(const std::string& e) {
  std::lock_guard<std::mutex> lk(mu_);
  if (error_.empty()) error_ = e;
}

std::string LayerFile::take_error() {
  std::lock_guard<std::mutex> lk(mu_);
  std::string e;
  e.swap(error_);
  return e;
}

long long LayerFile::bytes_read() const {
  std::lock_guard<std::mutex> lk(mu_);
  return bytes_read_;
}
double LayerFile::read_ms() const {
  std::lock_guard<std::mutex> lk(mu_);
  return read_ms_;
}

void LayerFile::reader_loop() {
  const int n = static_cast<int>(slots_.size());
  for (;;) {
    Req r;
    {
      std::unique_lock<std::mutex> lk(mu_);
      cv_req_.wait(lk, [&] { return stop_ || !queue_.empty(); });
      if (stop_) return;
      r = queue_.front();
      queue_.pop_front();
      // the slot's previous copy must have finished (released by the copy stream)
      const int k = static_cast<int>(r.seq % n);
      const bool freed = cv_free_.wait_for(lk, std::chrono::milliseconds(wait_ms_),
                                           [&] { return stop_ || released_[k] >= r.seq - n; });
      if (stop_) return;
      if (!freed && error_.empty()) error_ = "layer file: staging slot never released (wait limit)";
    }
    const int k = static_cast<int>(r.seq % n);
    std::string err;
    const auto t0 = std::chrono::steady_clock::now();
    const bool ok = pread_all(slots_[k], blob_, static_cast<long long>(r.layer) * stride_, err);
    ::posix_fadvise(fd_, static_cast<off_t>(r.layer) * static_cast<off_t>(stride_), static_cast<off_t>(stride_),
                    POSIX_FADV_DONTNEED);
    const double ms = std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - t0).count();
    {
      std::lock_guard<std::mutex> lk(mu_);
      if (!ok && error_.empty()) error_ = err;
      bytes_read_ += ok ? static_cast<long long>(blob_) : 0;
      read_ms_ += ms;
      ready_seq_ = r.seq;  // also on failure: the copy proceeds, the step reports the error
    }
    cv_ready_.notify_all();
  }
}

void CUDART_CB LayerFile::host_wait_read(void* arg) {
  Arg* a = static_cast<Arg*>(arg);
  LayerFile* f = a->f;
  {
    std::unique_lock<std::mutex> lk(f->mu_);
    const bool ok = f->cv_ready_.wait_for(lk, std::chrono::milliseconds(f->wait_ms_),
                                          [&] { return f->stop_ || f->ready_seq_ >= a->seq; });
    if (!ok && f->error_.empty()) f->error_ = "layer file: read did not finish (wait limit)";
  }
  delete a;
}

void CUDART_CB LayerFile::host_release(void* arg) {
  Arg* a = static_cast<Arg*>(arg);
  LayerFile* f = a->f;
  {
    std::lock_guard<std::mutex> lk(f->mu_);
    const int k = static_cast<int>(a->seq % static_cast<long long>(f->slots_.size()));
    f->released_[k] = a->seq;
  }
  f->cv_free_.notify_all();
  delete a;
}

cudaError_t LayerFile::stream_layer(int layer, void* dst, cudaStream_t copy_stream) {
  long long seq;
  {
    std::lock_guard<std::mutex> lk(mu_);
    seq = next_seq_++;
    queue_.push_back(Req{seq, layer});
  }
  cv_req_.notify_all();
  const int k = static_cast<int>(seq % static_cast<long long>(slots_.size()));
  cudaError_t e = cudaLaunchHostFunc(copy_stream, host_wait_read, new Arg{this, seq});
  if (e != cudaSuccess) return e;
  e = cudaMemcpyAsync(dst, slots_[k], blob_, cudaMemcpyHostToDevice, copy_stream);
  if (e != cudaSuccess) return e;
  return cudaLaunchHostFunc(copy_stream, host_release, new Arg{this, seq});
}

}  // namespace soup
