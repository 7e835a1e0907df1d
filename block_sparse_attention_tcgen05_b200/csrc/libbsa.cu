// Single translation unit for libbsa.so: the device status word is shared by every
// kernel without relocatable device code.
#include "common.cu"
#include "attention.cu"
