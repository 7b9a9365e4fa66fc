"""B200-native packed Delta-rule state decode step (sm_100a CUDA behind a C ABI).

The compute path is the shared library built from `csrc/` (`libstq.so`); the
Python module `stq` only marshals arguments to it. `workload` draws the seeded
synthetic inputs. `calibrate` sequences the library calls of the offline,
lifetime-aware width allocation; `diagnostics` runs the paired FP32 / quantised
error-lifetime check."""
