"""B200-native NVFP4 GPTQ + Schur Replay layer solve."""
