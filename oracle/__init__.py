"""Float64 CPU oracle for VDA forward.  Test infrastructure only: never imported by the product path."""
