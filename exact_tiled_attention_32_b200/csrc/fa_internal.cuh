// fa_internal.cuh -- host-side state shared by the translation units of
// libfa.so (not part of the C ABI).
#pragma once
#include <cuda.h>
#include <atomic>
#include <cstdint>

namespace fa_sm100 {

// Per-device set-up, done once on the first call on that device.
struct DeviceState {
    bool init = false;
    int status_code = FA_OK;
    int num_sms = 0;
    int* status = nullptr;        // device: [0] code, [1] wait site, [2] block
    unsigned long long* sched = nullptr;   // device: kSchedSlots work counters {epoch, items taken}
    std::atomic<unsigned> sched_seq{0};   // launches so far (picks the counter)
};

// Work counters per device: consecutive forward launches take consecutive
// counters, so launches running at the same time on different streams do not
// share one; a counter's epoch tells its launches apart.
constexpr int kSchedSlots = 64;

constexpr int kMaxDevices = 64;

// Sets up device `dev` (properties, the tensor-map encoder, the status word,
// the forward kernels' shared-memory limits); returns FA_OK or the error.
int init_device(int dev, DeviceState** out);

// 4-D tensor map with the given box, 128-byte swizzle; bf16 elements, or
// bytes (FP8) when `bytes` is set.
bool encode_map(CUtensorMap* m, const void* base, const uint64_t dims[4], const uint64_t strides[3],
                const uint32_t box[4], bool bytes = false);

}  // namespace fa_sm100
