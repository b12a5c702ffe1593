"""B200-native persistent op-queue runtime (GPUOS-style persistent execution).

Submodules:
  gpuos      -- ctypes binding of the C ABI in include/gpuos.h (libgpuos.so)
  workloads  -- seeded synthetic op streams (shared input generator)
  streams    -- builds gpuos descriptors for a workload on device arenas
  trace      -- host-side ordering audit of the device event log
  measure    -- algorithmic byte counts and roofline arithmetic
  replicas   -- one independent runtime per GPU under torch.distributed

Importing the package imports nothing else; the CUDA library is loaded on
first use of ``persistent_execution_b200.gpuos``.
"""
