// Host-side count of the kernel launches this library has enqueued, read
// through pq_launch_count(). Every launch site adds one right after its
// launch; the count is process-wide and covers all devices and threads.
#pragma once
#include <stdint.h>

#include <atomic>

namespace pqc {
extern std::atomic<int64_t> launches;
inline void count_launch() { launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace pqc
