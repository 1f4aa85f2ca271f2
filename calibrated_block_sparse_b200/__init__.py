"""CalibAtt hot path on B200 (sm_100a): C-ABI library libcalibatt.so and its ctypes binding."""
