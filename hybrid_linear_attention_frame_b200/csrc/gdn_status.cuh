// Device status word shared by the kernels of this library.  The library is
// compiled as one translation unit (gdn_lib.cu), so this definition is unique.
#pragma once

namespace gdn {
// 0 = fine; otherwise the first bounded wait that ran out records a nonzero code.
__device__ int g_device_status = 0;
}  // namespace gdn
