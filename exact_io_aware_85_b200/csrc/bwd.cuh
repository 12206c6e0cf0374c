// bwd.cuh — attention backward (placeholder until the kernels land).
#pragma once
#include "sm100.cuh"
