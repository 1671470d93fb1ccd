// Shared device-side includes for the vattn kernels (single translation
// unit: vattn.cu includes every kernel header).
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sm100.cuh"
