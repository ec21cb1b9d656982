// Process-wide runtime counters of the library.
#include <stdint.h>

#include <atomic>

namespace cp {

// Number of kernels the library has launched (all devices, all threads).
std::atomic<uint64_t>& launch_counter() {
  static std::atomic<uint64_t> n{0};
  return n;
}

}  // namespace cp
