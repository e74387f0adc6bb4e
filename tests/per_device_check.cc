// CPU check of PerDeviceOnce (head_attention_qk_b200/csrc/per_device.h), the
// per-device one-time kernel setup: compiled and run by
// tests/test_per_device.py with g++.  Devices are ordinals only; the "setup"
// here counts its runs instead of calling CUDA.
#include <atomic>
#include <chrono>
#include <cstdio>
#include <thread>
#include <vector>

#include "../head_attention_qk_b200/csrc/per_device.h"

#define CHECK(c)                                                   \
  do {                                                             \
    if (!(c)) {                                                    \
      std::fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #c); \
      return 1;                                                    \
    }                                                              \
  } while (0)

int main() {
  hattn::PerDeviceOnce once;
  std::atomic<int> runs[8];
  for (auto& r : runs) r = 0;

  // each device runs its setup once, independently of the others
  for (int rep = 0; rep < 3; ++rep)
    for (int d = 0; d < 4; ++d) CHECK(once.ensure(d, [&] { ++runs[d]; return true; }));
  for (int d = 0; d < 4; ++d) CHECK(runs[d] == 1);
  CHECK(runs[4] == 0);

  // a device set up on one ordinal is not set up on another: the second
  // device of a process sees its own first call
  CHECK(once.ensure(5, [&] { ++runs[5]; return true; }));
  CHECK(runs[5] == 1);

  // a failed setup is not remembered: the next call tries again
  CHECK(!once.ensure(6, [&] { ++runs[6]; return false; }));
  CHECK(!once.ensure(6, [&] { ++runs[6]; return false; }));
  CHECK(once.ensure(6, [&] { ++runs[6]; return true; }));
  CHECK(once.ensure(6, [&] { ++runs[6]; return true; }));
  CHECK(runs[6] == 3);

  // ordinals outside the table are refused without running the setup
  bool ran = false;
  CHECK(!once.ensure(-1, [&] { ran = true; return true; }));
  CHECK(!once.ensure(hattn::PerDeviceOnce::kMaxDevices, [&] { ran = true; return true; }));
  CHECK(!ran);

  // many host threads racing on first use of one device run the setup once
  std::atomic<int> racing{0};
  std::atomic<int> ok{0};
  std::vector<std::thread> ts;
  for (int t = 0; t < 16; ++t)
    ts.emplace_back([&] {
      if (once.ensure(7, [&] {
            ++racing;
            std::this_thread::sleep_for(std::chrono::milliseconds(20));
            return true;
          }))
        ++ok;
    });
  for (auto& t : ts) t.join();
  CHECK(racing == 1);
  CHECK(ok == 16);
  std::printf("per_device ok\n");
  return 0;
}
