// Fused tensor-core PISA attention (tcgen05 / TMEM / TMA) -- see below.
#pragma once
#include "common.cuh"
