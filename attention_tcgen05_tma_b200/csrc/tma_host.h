// Host-side access to the driver's tensor-map encoder, shared by every TMA kernel's launcher.
#pragma once

#include <cuda.h>

namespace hys {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled from the driver, looked up once per process (the first caller does the
// lookup; concurrent first calls are safe); nullptr when the driver does not provide it.
EncodeTiledFn tma_encode_fn();

}  // namespace hys
