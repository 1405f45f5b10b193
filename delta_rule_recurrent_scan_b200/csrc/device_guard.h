// Scoped switch of the calling thread's current CUDA device.
//
// Every entry point launches on the device that owns its state buffer.  The
// library links its own CUDA runtime, but the current device of a thread is
// the driver's current context, which the caller's runtime (PyTorch's, say)
// reads too; so an entry point that switched devices and left it switched
// would change the caller's current device.  ScopedDevice saves the current
// device when it first switches and puts it back when it goes out of scope,
// on every return path.
//
// The device calls are a template parameter so that the save / switch /
// restore logic can be checked on a host without a GPU against a fake
// (a header of its own, with no CUDA include).
#pragma once

namespace kdn {

// Ops must provide:  static int get(int* dev);  static int set(int dev);
// returning 0 on success (the cudaError_t convention).
template <class Ops>
class ScopedDevice {
 public:
  ScopedDevice() = default;
  ScopedDevice(const ScopedDevice&) = delete;
  ScopedDevice& operator=(const ScopedDevice&) = delete;
  ~ScopedDevice() { restore(); }

  // Make ``dev`` current.  The device that was current before the first switch is remembered
  // (once) and restored by restore() or the destructor.  Returns the error of the failing call.
  int switch_to(int dev) {
    int cur = -1;
    int e = Ops::get(&cur);
    if (e != 0) return e;
    if (cur == dev) return 0;
    if (!saved_) saved_ = true, prev_ = cur;
    return Ops::set(dev);
  }

  // Put the remembered device back (no-op when nothing was switched).  Returns the error of the call.
  int restore() {
    if (!saved_) return 0;
    saved_ = false;
    return Ops::set(prev_);
  }

  bool switched() const { return saved_; }

 private:
  bool saved_ = false;
  int prev_ = -1;
};

}  // namespace kdn
