// kvq_srft_d256.cu -- the SRFT codec kernels at D = 256 (see kvq_srft.cuh).
#define KVQ_SRFT_D 256
#include "kvq_srft.cuh"
