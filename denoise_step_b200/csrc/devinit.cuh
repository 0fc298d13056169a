// Per-device set-up shared by the host code of the library: a status word for
// calls made without a context, the SM count, and a once-per-device guard for
// kernel attributes (all keyed by the current CUDA device).
#pragma once
#include <cstdint>

namespace pl {

constexpr int kMaxDevices = 64;

// Current device, or -1 when it cannot be read or is beyond kMaxDevices.
int current_device();
// Device address (on the current device) of the library's status word for
// context-free calls; null when the lookup fails. The first call on a device
// looks the address up (cudaGetSymbolAddress): make it outside stream capture.
uint32_t* call_status_word();
// Streaming multiprocessors of the current device (148 if it cannot be read).
int device_sms();

}  // namespace pl
