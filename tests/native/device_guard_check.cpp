// Host-only check of kdn::ScopedDevice against a fake device API (no GPU, no CUDA headers).
// Exit status 0 when every check holds; the failing check is printed otherwise.
#include <cstdio>

#include "device_guard.h"

namespace {

int g_current = 0;      // the fake thread's current device
int g_sets = 0;         // set() calls made
int g_fail_get = 0;     // error code get() returns (0 = success)
int g_fail_set_to = -1; // set(dev) fails with code 7 for this device

struct FakeOps {
  static int get(int* dev) {
    if (g_fail_get) return g_fail_get;
    *dev = g_current;
    return 0;
  }
  static int set(int dev) {
    ++g_sets;
    if (dev == g_fail_set_to) return 7;
    g_current = dev;
    return 0;
  }
};

using Guard = kdn::ScopedDevice<FakeOps>;
int g_failures = 0;

void check(bool ok, const char* what) {
  if (!ok) {
    std::printf("FAILED: %s\n", what);
    ++g_failures;
  }
}

void reset(int cur) { g_current = cur, g_sets = 0, g_fail_get = 0, g_fail_set_to = -1; }

// An entry point that switches to ``dev`` and returns early or late.
int entry(int dev, bool early) {
  Guard g;
  int e = g.switch_to(dev);
  if (e != 0) return e;
  if (early) return 1;
  check(g_current == dev, "inside the call the state's device is current");
  return 0;
}

}  // namespace

int main() {
  reset(0);
  { Guard g; }
  check(g_sets == 0 && g_current == 0, "a guard that never switched leaves the device alone");

  reset(0);
  check(entry(0, false) == 0 && g_sets == 0, "same device: no set() at all");

  reset(0);
  entry(3, false);
  check(g_current == 0, "switched to 3 and back to 0 on a normal return");
  check(g_sets == 2, "exactly one switch and one restore");

  reset(2);
  entry(5, true);
  check(g_current == 2, "restored on an early return");

  reset(1);
  {
    Guard g;
    g.switch_to(4);
    g.switch_to(6);  // a second switch keeps the first saved device
    check(g_current == 6, "second switch takes effect");
  }
  check(g_current == 1, "the device current before the first switch is the one restored");

  reset(1);
  {
    Guard g;
    g.switch_to(4);
    check(g.restore() == 0 && g_current == 1, "explicit restore");
    check(!g.switched(), "nothing left to restore");
  }
  check(g_current == 1 && g_sets == 2, "the destructor does not restore twice");

  reset(0);
  g_fail_get = 5;
  check(entry(3, false) == 5 && g_current == 0 && g_sets == 0, "a failing get() is reported and nothing is set");

  reset(0);
  g_fail_set_to = 3;
  check(entry(3, false) == 7, "a failing set() is reported");
  check(g_current == 0, "the device is unchanged after a failed switch");

  if (g_failures == 0) std::printf("ok\n");
  return g_failures == 0 ? 0 : 1;
}
