// The library as one translation unit: the layer step, its optimizer and
// building blocks (gptlayer.cu), then the extensions that use the same
// argument checks, device check and launch recorder: gradient clipping and
// accumulation (optim_ext.cuh) and stacks of layers (stack_ext.cuh).
#include "gptlayer.cu"
#include "optim_ext.cuh"
#include "stack_ext.cuh"
