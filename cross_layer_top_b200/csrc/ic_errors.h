// Error codes shared by host and device code of libindexcache.
#pragma once

#include "../../include/indexcache.h"

namespace ic {
// Values latched in the context's device error word (first one wins).
enum DeviceError : int {
    kDevOk = 0,
    kDevTimeoutProducer = 1,
    kDevTimeoutMma = 2,
    kDevTimeoutEpilogue = 3,
    kDevSmemMisaligned = 4,
    kDevBadIndex = 5,
    kDevTimeoutDrain = 6,
};
}  // namespace ic
