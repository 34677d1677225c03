// host_util.h -- per-device host state of the library: one-time kernel set-up
// (shared-memory and cluster attributes, occupancy queries) and the device's
// SM count.  Kernel attributes are per device, so each is applied once on
// every device the library is used on; std::call_once makes that safe when
// several host threads call in at once.
#pragma once
#include <cuda_runtime.h>

#include <mutex>

namespace csa2 {

constexpr int kMaxDevices = 64;

inline int current_device() {
    int d = -1;
    if (cudaGetDevice(&d) != cudaSuccess) {
        (void)cudaGetLastError();
        return -1;
    }
    return d;
}

// Runs a set-up function once per device, with that device current; later
// calls on the same device return the first call's result.
struct DeviceOnce {
    std::once_flag flag[kMaxDevices];
    cudaError_t err[kMaxDevices] = {};

    template <class F>
    cudaError_t run(F&& f) {
        const int d = current_device();
        if (d < 0 || d >= kMaxDevices) return cudaErrorInvalidDevice;
        std::call_once(flag[d], [&] { err[d] = f(); });
        return err[d];
    }
};

// A per-device value computed once by f() (for example an occupancy figure).
template <class T>
struct DeviceValue {
    DeviceOnce once;
    T value[kMaxDevices] = {};

    template <class F>
    T get(F&& f, T fallback) {
        const int d = current_device();
        if (d < 0 || d >= kMaxDevices) return fallback;
        once.run([&] {
            value[d] = f();
            return cudaSuccess;
        });
        return value[d];
    }
};

// Streaming multiprocessors of the current device (148 on B200).
inline int device_sm_count() {
    static DeviceValue<int> sms;
    return sms.get(
        [] {
            int n = 0;
            if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, current_device()) != cudaSuccess) {
                (void)cudaGetLastError();
                n = 0;
            }
            return n;
        },
        0);
}

}  // namespace csa2
