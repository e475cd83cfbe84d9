"""B200-native (sm_100a) training step of one GPT transformer layer with
Megatron-style tensor parallelism on a single GPU.

  gptlayer  ctypes binding of libgptlayer.so (the C ABI in include/)
  harness   torch-held device memory and the four calls of one step
  synth     seeded synthetic inputs (shared with the tests' CPU oracle)
  build     nvcc build of the library for sm_100a
"""
