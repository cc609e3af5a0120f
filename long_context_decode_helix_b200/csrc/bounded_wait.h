// bounded_wait.h -- a host-side wait with a wall-clock limit (header-only, no CUDA dependency).
//
// The library's device-side waits all give up after a limit (mbarrier polls read %globaltimer);
// this is the host-side counterpart: instead of blocking in cudaStreamSynchronize for as long as
// the GPU takes, a caller polls a completion query until it reports done, reports an error, or
// the limit passes. The query is a template argument so the loop can be exercised on a machine
// without a GPU with a fake query (one that never completes, one that fails).
#pragma once

#include <chrono>
#include <stdint.h>
#include <thread>

#include "helix.h"

namespace helix {

// Result of one poll of the awaited work.
enum class PollResult { kDone, kPending, kError };

// Polls `query()` until it returns kDone (HELIX_OK) or kError (HELIX_ERR_CUDA), or until `limit_us`
// microseconds of steady-clock time have passed since the first poll (HELIX_ERR_TIMEOUT). The
// first few polls are back to back; after that the thread yields between polls and, once the
// wait has lasted a millisecond, sleeps 50 us between them so a long wait does not burn a core.
template <class Query>
helix_status poll_with_limit(Query&& query, uint64_t limit_us) {
  using clock = std::chrono::steady_clock;
  const auto t0 = clock::now();
  const auto limit = std::chrono::microseconds(limit_us);
  for (uint64_t n = 0;; ++n) {
    switch (query()) {
      case PollResult::kDone: return HELIX_OK;
      case PollResult::kError: return HELIX_ERR_CUDA;
      case PollResult::kPending: break;
    }
    const auto waited = clock::now() - t0;
    if (waited >= limit) return HELIX_ERR_TIMEOUT;
    if (n < 64) continue;
    if (waited < std::chrono::milliseconds(1))
      std::this_thread::yield();
    else
      std::this_thread::sleep_for(std::chrono::microseconds(50));
  }
}

}  // namespace helix
