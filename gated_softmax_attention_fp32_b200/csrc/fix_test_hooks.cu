// Test hooks, compiled only into the test build of the library
// (libfixattn_test.so, -DFIX_TEST_HOOKS); the product library has none.
//
// fix_attn_test_stall_forward(1) makes every following tensor-core forward
// launch run "stalled": its producer warp issues no loads, so nothing is ever
// in flight, and every bounded wait gives up after 1 ms instead of 1 s.  The
// kernel must then take its abort path -- record FIX_ERR_DEVICE_TIMEOUT in the
// status word, leave every role, release TMEM -- and the next ordinary call
// must succeed.  This exercises the device-side failure detection without a
// GPU fault or a hang.
#ifdef FIX_TEST_HOOKS
#include <atomic>

#include "fix_internal.h"

namespace fix {
static std::atomic<int> g_stall{0};
int test_stall_forward() { return g_stall.load(); }
}  // namespace fix

extern "C" void fix_attn_test_stall_forward(int on) { fix::g_stall.store(on ? 1 : 0); }
#endif
