"""Hardware-rate probes for the GEMM kernels' design: standalone CUDA programs
that time one mechanism each on the B200 (int8 MMA issue rates, L2 -> shared
memory bulk copies, TMEM loads and stores, the FP32 / conversion pipes, TMEM
traffic beside the MMA).  They are measurement programs, not part of the
library; `python -m bit_group_quantized_flexq_b200.probes.run` builds and runs
them."""
