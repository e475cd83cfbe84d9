// The library as one translation unit: the layer step, its optimizer and
// building blocks (gptlayer.cu), then the optimizer extensions that use the
// same argument checks, device check and launch recorder (optim_ext.cuh:
// gradient clipping by global norm, gradient accumulation).
#include "gptlayer.cu"
#include "optim_ext.cuh"
