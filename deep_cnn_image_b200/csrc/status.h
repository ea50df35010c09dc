// status.h -- bits of the handle's sticky device status word.
#pragma once

namespace alx {

constexpr int STATUS_TIMEOUT = 1 << 0;      // a bounded device wait ran out
constexpr int STATUS_LABEL_RANGE = 1 << 1;  // a label outside [0, classes)
constexpr int STATUS_BAD_LAUNCH = 1 << 2;   // a kernel was given a shape it cannot serve

}  // namespace alx
