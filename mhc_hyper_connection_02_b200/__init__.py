"""mHC (HC=4) pre-map / post-map on B200: Python binding of the ``libmhc.so`` C ABI."""
